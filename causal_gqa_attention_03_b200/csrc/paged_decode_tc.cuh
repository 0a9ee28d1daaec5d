// The paged-KV decode step on the tensor cores, head dimension 64 or 128.
//
// Same operation, items, chunk stream, partial slots and merge as
// paged_decode.cuh; here the two contractions of a 128-token chunk run as
// tcgen05 MMAs with the item's query heads as a narrow dimension of 16:
//   S^T[t, h] = K[t, :] . q[h, :]       A = K chunk (M = 128 tokens, K-major),
//                                        B = q rows (N = 16, K-major, rows >= GT zero)
// and, at d = 128,
//   O^T[c, h] += sum_t V[t, c] P^T[h, t] A = V chunk (M = 128 columns, MN-major),
//                                        B = P^T (N = 16, K = 128 tokens, K-major)
// or, at d = 64 (an M of 64 columns would need another accumulator layout),
//   O[h, c] += sum_t P[h, t] V[t, c]    A = P (M = 128 rows, rows >= GT zero,
//                                        K = 128 tokens, K-major), B = V chunk
//                                        (N = 64 columns, MN-major),
// both accumulating in tensor memory.  The FP32 pipes keep only the softmax
// (a thread per token), so the step stays bound by HBM.
//
// Layout of a K or V chunk in shared memory: 16 atoms of 8 tokens.  At
// d = 128 an atom is [columns 0-63: 8 rows x 128 B][columns 64-127: 8 rows x
// 128 B] (2 KB, the 128-byte swizzle inside each 1 KB half), and one 4-D TMA
// box (64 columns x 8 rows x 2 halves x R/8 atoms, the tensor viewed with row
// stride 256 B, half stride 128 B and atom stride 2 KB) brings a whole page of
// R tokens.  At d = 64 an atom is 8 rows x 128 B (1 KB), and a 2-D box of R
// rows brings the page.  The MMA descriptors read either with an 8-row stride
// of one atom.
//
// Roles (224 threads): warps 0-3 softmax (thread = token for S^T; thread =
// column for O^T at d = 128, warp 0's lanes = query rows for O at d = 64),
// warp 4 issues the MMAs, warps 5 and 6 produce the K and the V ring.  Rings:
// K (+ the q rows) in NK stages, released when S^T is done; V in NV stages,
// released when the chunk's P.V is done.  S^T is double buffered in tensor
// memory; P is two shared-memory tiles, alternating, so a chunk's softmax
// overlaps the previous chunk's P.V.  Online softmax across a segment's chunks with a lazy maximum:
// the running max moves only when a chunk's max exceeds it by more than 2^8,
// and O is rescaled only then.
#pragma once

#include "paged_decode.cuh"

namespace tessera {

constexpr int kDecTcThreads = 224;
constexpr int kDecTcMmaWarp = 4;
constexpr int kDecTcTmaWarp = 5;   // K (and q) producer; warp 6 produces V
constexpr int kDecTcN = 16;              // N of both products: query heads per item, padded
constexpr float kDecTcRescale = 8.0f;    // log2 units

template <int D_>
struct DecTcCfg {
  static constexpr int D = D_;
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int CH = kDecodeChunk;       // 128 tokens
  static constexpr int HALVES = D / 64;         // 64-column halves of a cache row
  static constexpr int ATOM = 1024 * HALVES;    // 8 tokens x D columns
  static constexpr int QHALF = kDecTcN * 128;   // one [16 rows][64 cols] bf16 sub-tile
  static constexpr int K_BYTES = (CH / 8) * ATOM;
  static constexpr int KSTAGE = K_BYTES + HALVES * QHALF;  // K, then the q rows
  static constexpr int VSTAGE = (CH / 8) * ATOM;
  static constexpr int NK = (D == 128) ? 3 : 4, NV = NK;
  // P: at d = 128 P^T [16 heads][128 tokens], at d = 64 P [128 rows][128
  // tokens]; either as two 64-token halves of PROWS rows x 128 B.  Two
  // buffers, alternating over a segment's good chunks.
  static constexpr int PROWS = (D == 128) ? kDecTcN : 128;
  static constexpr int PHALF = PROWS * 128;
  static constexpr int PBUF = 2 * PHALF;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NK * KSTAGE;
  static constexpr int P_OFF = V_OFF + NV * VSTAGE;
  static constexpr int RED_OFF = P_OFF + 2 * PBUF;     // float [2][4][16] chunk maxima
  static constexpr int LRED_OFF = RED_OFF + 512;       // float [4][16] row-sum partials
  static constexpr int SMETA_OFF = LRED_OFF + 256;     // int [2][8] (per S^T buffer)
  static constexpr int KMETA_OFF = SMETA_OFF + 64;     // int [NK][8] (per K stage)
  static constexpr int BAR_OFF = KMETA_OFF + 32 * NK;
  // full_k[NK], empty_k[NK], full_v[NV], empty_v[NV], s_full[2], s_free[2],
  // p_full[2], pv_done[2], drain
  static constexpr int NBAR = 2 * NK + 2 * NV + 9;
  static constexpr int SLOT_OFF = BAR_OFF + 8 * NBAR;
  static constexpr int BYTES = SLOT_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr int S_COL = 0;   // two buffers of 16 columns
  static constexpr int O_COL = 32;  // O^T: 16 columns (d = 128); O: 64 columns (d = 64)
  static constexpr uint32_t TMEM_COLS = (D == 128) ? 64 : 128;
  static_assert(KSTAGE % 1024 == 0 && VSTAGE % 1024 == 0 && P_OFF % 1024 == 0, "alignment");
  static_assert(SMEM <= 232448, "fits the 227 KB a CTA may use");
};

// 16-byte units to add to a K-major 128-byte-swizzled descriptor for K step
// kk (16 elements) when the operand's two 64-column sub-tiles are `sub` bytes
// apart.
__device__ __forceinline__ uint32_t kmajor_step(int kk, int sub) {
  return static_cast<uint32_t>((kk >> 2) * (sub >> 4) + (kk & 3) * 2);
}

// Producer warps, one per ring.  Each finds this CTA's share [lo, hi) of the
// chunk stream from the lengths and walks it chunk by chunk, one ring stage
// per chunk, reading the block ids of the next chunk while the current one is
// issued: a chunk's pages are TMA boxes of R = min(bs, 128) rows, evict-first
// in L2.  The K warp (is_v false) fills the K ring, with the q rows fetched
// by TMA with every K chunk, and ends it with a sentinel stage (b = -1); the
// V warp fills the V ring.
template <int D, int GT>
__device__ __forceinline__ void dectc_produce(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              const CUtensorMap* tm_q, const DecodeParams& p,
                                              uint8_t* sm, int* kmeta, uint64_t* full_k,
                                              uint64_t* empty_k, uint64_t* full_v,
                                              uint64_t* empty_v, int lane, bool is_v) {
  using C = DecTcCfg<D>;
  const int R = p.rows_per_box;
  const long long HZ = static_cast<long long>(p.Hkv) * p.zgroups;
  long long tot = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    long long ch = b < p.B ? decode_chunks(decode_len(p, b)) : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ch += __shfl_xor_sync(0xffffffffu, ch, off);
    tot += ch;
  }
  const long long total = tot * HZ;
  const long long per = (total + gridDim.x - 1) / gridDim.x;
  const long long lo = static_cast<long long>(blockIdx.x) * per;
  long long hi = min(lo + per, total);
  uint32_t produced = 0;
  bool alive = true;
  if (lo < hi) {
    DecodeCursor cur{};
    long long pre = 0;
    for (int b0 = 0;; b0 += 32) {
      const int b = b0 + lane;
      const int n = b < p.B ? decode_len(p, b) : 0;
      const long long ch = static_cast<long long>(decode_chunks(n)) * HZ;
      const long long incl = warp_incl_scan(ch, lane) + pre;
      const unsigned hit = __ballot_sync(0xffffffffu, b < p.B && incl > lo);
      if (hit) {
        const int j = __ffs(hit) - 1;
        cur.b = b0 + j;
        cur.n = __shfl_sync(0xffffffffu, n, j);
        const long long start_b = __shfl_sync(0xffffffffu, incl - ch, j);
        cur.nchunks = decode_chunks(cur.n);
        const long long r = lo - start_b;
        cur.gz = static_cast<int>(r / cur.nchunks);
        cur.c = static_cast<int>(r % cur.nchunks);
        cur.item0 = start_b + static_cast<long long>(cur.gz) * cur.nchunks;
        cur.slot = static_cast<int>(blockIdx.x - cur.item0 / per);
        break;
      }
      pre = __shfl_sync(0xffffffffu, incl, 31);
    }
    const uint64_t pol = ptx::policy_evict_first();
    const uint64_t keep = ptx::policy_evict_last();
    // The producer loop's own latency bounds the step at d = 64, where a
    // chunk is half the bytes: there R and the block size (powers of two) are
    // used as shifts and each item's slot is computed once.  At d = 128 the
    // step is bound by HBM, and the same changes measured 2-3 % slower on
    // the serving batch, so that path keeps the divisions.
    constexpr bool kLean = D == 64;
    const int lg_r = 31 - __clz(R), lg_bs = 31 - __clz(p.bs);
    auto load_ids = [&](const DecodeCursor& cu, int& blk, int& npg) {
      const int nt = min(C::CH, cu.n - cu.c * C::CH);
      npg = kLean ? (nt + R - 1) >> lg_r : (nt + R - 1) / R;
      blk = 0;
      if (lane < npg)
        blk = p.block_table[static_cast<long long>(cu.b) * p.max_blocks +
                            (kLean ? (cu.c * C::CH + lane * R) >> lg_bs
                                   : (cu.c * C::CH + lane * R) / p.bs)];
    };
    auto page_row = [&](int tok) {  // token tok's row within its cache block
      return kLean ? (tok & (p.bs - 1)) : tok % p.bs;
    };
    int blk, npg;
    load_ids(cur, blk, npg);
    for (long long pos = lo; pos < hi; ++pos) {
      DecodeCursor nxt = cur;
      int nblk = 0, nnpg = 0;
      if (pos + 1 < hi) {
        if (++nxt.c == nxt.nchunks) {
          nxt.c = 0;
          nxt.item0 += nxt.nchunks;
          nxt.slot = static_cast<int>(blockIdx.x - nxt.item0 / per);
          if (++nxt.gz == HZ) {
            nxt.gz = 0;
            do {  // the stream has more chunks, so such a sequence exists before B
              ++nxt.b;
              nxt.n = nxt.b < p.B ? decode_len(p, nxt.b) : -1;
            } while (nxt.n == 0);
            if (nxt.n < 0) {  // lengths changed under the kernel: stop after this chunk
              decode_error(p, kErrDecodeInput);
              nxt.n = 0;
            }
            nxt.nchunks = decode_chunks(nxt.n);
          }
        }
        if (nxt.n > 0)
          load_ids(nxt, nblk, nnpg);
        else
          hi = pos + 1;
      }
      const bool bad = __any_sync(0xffffffffu, lane < npg && (blk < 0 || blk >= p.num_blocks));
      const bool seg_first = pos == lo || cur.c == 0;
      const bool item_last = cur.c == cur.nchunks - 1;
      const bool seg_last = pos == hi - 1 || item_last;
      const int flags = (bad ? kStageBad : 0) | (seg_first ? kStageSegFirst : 0) |
                        (seg_last ? kStageSegLast : 0) | (item_last ? kStageItemLast : 0);
      const int nt = min(C::CH, cur.n - cur.c * C::CH);
      const int g = cur.gz / p.zgroups, z = cur.gz % p.zgroups;
      const int tok0 = cur.c * C::CH;
      if (!is_v) {
        // ---- K and the q rows
        const uint32_t sk = produced % C::NK;
        bool ok = true;
        if (lane == 0) {
          if (bad) decode_error(p, kErrDecodeInput);
          ok = decode_wait(&empty_k[sk], ((produced / C::NK) & 1) ^ 1u);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) decode_error(p, kErrDecodeWait);
          alive = false;
          break;
        }
        uint8_t* kst = sm + C::K_OFF + sk * C::KSTAGE;
        if (lane == 0) {
          int* m = kmeta + 8 * sk;
          m[0] = cur.b;
          m[1] = cur.gz;
          m[2] = cur.c;
          m[3] = nt;
          m[4] = flags;
          m[5] = kLean ? cur.slot : static_cast<int>(blockIdx.x - cur.item0 / per);
          if (bad) {
            ptx::mbar_arrive(&full_k[sk]);
          } else {
            ptx::mbar_arrive_expect_tx(&full_k[sk],
                                       static_cast<uint32_t>(npg * R * 2 * D + GT * 2 * D));
            const int qrow = (cur.b * p.Hq + g * p.G + z * GT);
#pragma unroll
            for (int h = 0; h < C::HALVES; ++h)
              ptx::tma_load_2d_hint(kst + C::K_BYTES + h * C::QHALF, tm_q, &full_k[sk], 64 * h,
                                    qrow, keep);
          }
        }
        __syncwarp();
        if (!bad && lane < npg) {
          const int row = (blk * p.Hkv + g) * p.bs + page_row(tok0 + lane * R);  // multiple of 8
          if constexpr (D == 128)
            ptx::tma_load_4d_hint(kst + lane * R * 256, tm_k, &full_k[sk], 0, 0, 0, row >> 3, pol);
          else
            ptx::tma_load_2d_hint(kst + lane * R * 128, tm_k, &full_k[sk], 0, row, pol);
        }
      } else {
        // ---- V
        const uint32_t sv = produced % C::NV;
        bool ok = true;
        if (lane == 0) ok = decode_wait(&empty_v[sv], ((produced / C::NV) & 1) ^ 1u);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) decode_error(p, kErrDecodeWait);
          alive = false;
          break;
        }
        uint8_t* vst = sm + C::V_OFF + sv * C::VSTAGE;
        if (lane == 0) {
          if (bad)
            ptx::mbar_arrive(&full_v[sv]);
          else
            ptx::mbar_arrive_expect_tx(&full_v[sv], static_cast<uint32_t>(npg * R * 2 * D));
        }
        __syncwarp();
        if (!bad && lane < npg) {
          const int row = (blk * p.Hkv + g) * p.bs + page_row(tok0 + lane * R);  // multiple of 8
          if constexpr (D == 128)
            ptx::tma_load_4d_hint(vst + lane * R * 256, tm_v, &full_v[sv], 0, 0, 0, row >> 3, pol);
          else
            ptx::tma_load_2d_hint(vst + lane * R * 128, tm_v, &full_v[sv], 0, row, pol);
        }
      }
      ++produced;
      cur = nxt;
      blk = nblk;
      npg = nnpg;
    }
  }
  if (alive && !is_v && lane == 0) {
    const uint32_t sk = produced % C::NK;
    if (decode_wait(&empty_k[sk], ((produced / C::NK) & 1) ^ 1u)) {
      kmeta[8 * sk] = -1;
      ptx::mbar_arrive(&full_k[sk]);
    } else {
      decode_error(p, kErrDecodeWait);
    }
  }
}

template <int D, int GT>
__global__ void __launch_bounds__(kDecTcThreads, 1)
    paged_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_q, const DecodeParams p) {
  static_assert(GT == 1 || GT == 2 || GT == 4 || GT == 8 || GT == 16, "heads per item");
  using C = DecTcCfg<D>;
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  float* red = reinterpret_cast<float*>(sm + C::RED_OFF);
  float* lred = reinterpret_cast<float*>(sm + C::LRED_OFF);
  int* smeta = reinterpret_cast<int*>(sm + C::SMETA_OFF);
  int* kmeta = reinterpret_cast<int*>(sm + C::KMETA_OFF);
  uint64_t* full_k = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* empty_k = full_k + C::NK;
  uint64_t* full_v = empty_k + C::NK;
  uint64_t* empty_v = full_v + C::NV;
  uint64_t* s_full = empty_v + C::NV;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;   // [2], per P buffer
  uint64_t* pv_done = p_full + 2;  // [2], per P buffer
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::SLOT_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp < 4) {
    // zero the q rows >= GT of every K stage and the P tile (never written
    // again: TMA writes rows < GT, the softmax heads < GT)
    for (int s = 0; s < C::NK; ++s)
      for (int i = tid; i < C::HALVES * C::QHALF / 16; i += 128)
        reinterpret_cast<uint4*>(sm + C::K_OFF + s * C::KSTAGE + C::K_BYTES)[i] =
            make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid; i < 2 * C::PBUF / 16; i += 128)
      reinterpret_cast<uint4*>(sm + C::P_OFF)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async_smem();
  } else if (warp == kDecTcMmaWarp) {
    if (lane == 0) {
      for (int s = 0; s < C::NK; ++s) {
        ptx::mbar_init(&full_k[s], 1);
        ptx::mbar_init(&empty_k[s], 1);
      }
      for (int s = 0; s < C::NV; ++s) {
        ptx::mbar_init(&full_v[s], 1);
        ptx::mbar_init(&empty_v[s], 1);
      }
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&s_full[b], 1);
        ptx::mbar_init(&s_free[b], 128);
      }
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&p_full[b], 128);
        ptx::mbar_init(&pv_done[b], 1);
      }
      ptx::mbar_init(drain, 1);
      ptx::fence_mbar_init();
    }
    __syncwarp();
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  } else if (lane == 0) {
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    ptx::prefetch_tensormap(&tm_q);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kDecTcTmaWarp || warp == kDecTcTmaWarp + 1) {
    dectc_produce<D, GT>(&tm_k, &tm_v, &tm_q, p, sm, kmeta, full_k, empty_k, full_v, empty_v,
                         lane, warp == kDecTcTmaWarp + 1);
  } else if (warp == kDecTcMmaWarp) {
    // ======================= MMA issue (lane 0; the warp waits) ===========
    const bool leader = lane == 0;
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, kDecTcN, false, false);
    // d = 128: O^T = V^T P^T (A MN-major); d = 64: O = P V (B MN-major)
    constexpr uint32_t kIdescO = D == 128 ? ptx::idesc_bf16_f32(128, kDecTcN, true, false)
                                          : ptx::idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t kHi = ptx::sdesc_sw128_hi(1024);      // q, P: 8-row groups 1 KB apart
    constexpr uint32_t kHiKV = ptx::sdesc_sw128_hi(C::ATOM); // K, V: 8-token atoms ATOM apart
    const uint32_t k_base = ptx::smem_u32(sm + C::K_OFF);
    const uint32_t v_base = ptx::smem_u32(sm + C::V_OFF);
    const uint32_t p_lo0 = ptx::sdesc_sw128_lo(ptx::smem_u32(sm + C::P_OFF), 16);
    bool pending = false;   // a good chunk whose P.V is still to issue
    uint32_t pend_sv = 0, pend_kc = 0, pend_acc = 0;
    uint32_t npv = 0;       // P.V products issued: buffer npv & 1, phase npv >> 1
    bool seg_good = false;  // the current segment has had a good chunk
    bool ok = true;
    // Each step handles chunk kc (its S^T, or nothing for a dropped chunk) and
    // the previous good chunk's P.V, in whichever order their inputs arrive,
    // so a late K chunk does not hold back the P.V that frees a V stage.
    auto ready = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, ptx::mbar_test_wait(bar, parity));
    };
    for (uint32_t kc = 0; ok; ++kc) {
      const uint32_t sk = kc % C::NK, buf = kc & 1;
      bool s_done = false, sentinel = false, bad = false;
      int m[8];
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!s_done || pending) {
        bool progressed = false;
        if (pending && ready(&p_full[npv & 1], (npv >> 1) & 1) &&
            ready(&full_v[pend_sv], (pend_kc / C::NV) & 1)) {
          ptx::tc_fence_after();
          if (leader) {
            const uint32_t p_lo = p_lo0 + (npv & 1) * (C::PBUF >> 4);
            // V (MN-major): 8-token atoms one ATOM apart (SBO), at d = 128 the
            // two 64-column halves 1 KB apart (LBO); K step kk = 16 tokens =
            // two atoms.  P (K-major): K step by kmajor_step over its halves.
            const uint32_t va = ptx::sdesc_sw128_lo(v_base + pend_sv * C::VSTAGE, C::ATOM / 2);
            if constexpr (D == 128) {
              ptx::mma_ss_lohi_rt(tmem + C::O_COL, va, kHiKV, p_lo, kHi, kIdescO, pend_acc);
#pragma unroll
              for (int kk = 1; kk < C::CH / 16; ++kk)
                ptx::mma_ss_lohi<1>(tmem + C::O_COL, va + kk * ((2 * C::ATOM) >> 4), kHiKV,
                                    p_lo + kmajor_step(kk, C::PHALF), kHi, kIdescO);
            } else {
              ptx::mma_ss_lohi_rt(tmem + C::O_COL, p_lo, kHi, va, kHiKV, kIdescO, pend_acc);
#pragma unroll
              for (int kk = 1; kk < C::CH / 16; ++kk)
                ptx::mma_ss_lohi<1>(tmem + C::O_COL, p_lo + kmajor_step(kk, C::PHALF), kHi,
                                    va + kk * ((2 * C::ATOM) >> 4), kHiKV, kIdescO);
            }
            ptx::tc_commit(&empty_v[pend_sv]);
            ptx::tc_commit(&pv_done[npv & 1]);
          }
          __syncwarp();
          ++npv;
          pending = false;
          progressed = true;
        }
        if (!s_done && ready(&full_k[sk], (kc / C::NK) & 1) &&
            ready(&s_free[buf], ((kc >> 1) & 1) ^ 1u)) {
#pragma unroll
          for (int i = 0; i < 8; ++i) m[i] = kmeta[8 * sk + i];
          if (leader) {
#pragma unroll
            for (int i = 0; i < 8; ++i) smeta[8 * buf + i] = m[i];
          }
          __syncwarp();
          s_done = true;
          progressed = true;
          if (m[0] < 0) {
            sentinel = true;  // passed on once the last P.V is issued
          } else if (m[4] & kStageBad) {
            bad = true;
            // nothing to multiply: hand the stages back in order
            ok = __all_sync(0xffffffffu, decode_wait(&full_v[kc % C::NV], (kc / C::NV) & 1));
            if (!ok) break;
            if (leader) {
              ptx::mbar_arrive(&empty_k[sk]);
              ptx::mbar_arrive(&empty_v[kc % C::NV]);
              ptx::mbar_arrive(&s_full[buf]);
            }
            __syncwarp();
          } else {
            ptx::tc_fence_after();
            if (leader) {
              // S^T = K q^T: A = K (K-major, column halves 1 KB apart, atoms 2 KB
              // apart), B = q rows (K-major, column halves 2 KB apart)
              const uint32_t ka = ptx::sdesc_sw128_lo(k_base + sk * C::KSTAGE, 16);
              const uint32_t qb = ptx::sdesc_sw128_lo(k_base + sk * C::KSTAGE + C::K_BYTES, 16);
              const uint32_t sd = tmem + C::S_COL + kDecTcN * buf;
              ptx::mma_ss_lohi<0>(sd, ka, kHiKV, qb, kHi, kIdescS);
#pragma unroll
              for (int kk = 1; kk < C::D / 16; ++kk)
                ptx::mma_ss_lohi<1>(sd, ka + kmajor_step(kk, C::ATOM / 2), kHiKV,
                                    qb + kmajor_step(kk, C::QHALF), kHi, kIdescS);
              ptx::tc_commit(&s_full[buf]);
              ptx::tc_commit(&empty_k[sk]);
            }
            __syncwarp();
          }
        }
        if (!progressed && ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (sentinel) {
        if (leader) ptx::mbar_arrive(&s_full[buf]);
        __syncwarp();
        break;
      }
      if (!bad) {
        pending = true;
        pend_sv = kc % C::NV;
        pend_kc = kc;
        pend_acc = seg_good ? 1u : 0u;
        seg_good = true;
      }
      if (m[4] & kStageSegLast) seg_good = false;
    }
    if (!ok) decode_error(p, kErrDecodeWait);
    // every MMA issued must finish before tensor memory is released
    if (leader) ptx::tc_commit(drain);
    __syncwarp();
    decode_wait(drain, 0);
    // and the softmax warps are done with it
    ptx::bar_sync_named(2, 160);
    ptx::tc_fence_after();
    __syncwarp();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  } else {
    // ======================= softmax (warps 0-3, thread = token) ===========
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::O_COL;
    const int t = tid;  // token of S^T, column of O^T
    float m_run[GT], l_w[GT];
#pragma unroll
    for (int gh = 0; gh < GT; ++gh) {
      m_run[gh] = -INFINITY;
      l_w[gh] = 0.f;
    }
    bool seg_good = false;
    uint32_t ngood = 0;  // good chunks seen: P buffer ngood & 1, phase ngood >> 1
    const uint32_t p_base = ptx::smem_u32(sm + C::P_OFF);
    for (uint32_t kc = 0;; ++kc) {
      const uint32_t buf = kc & 1;
      bool ok = decode_wait(&s_full[buf], (kc >> 1) & 1);
      ok = ptx::bar_red_and(1, 128, ok);
      if (!ok) {
        if (tid == 0) decode_error(p, kErrDecodeWait);
        break;
      }
      int m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = smeta[8 * buf + i];
      if (m[0] < 0) break;  // sentinel
      const int flags = m[4], nt = m[3];
      const bool bad = (flags & kStageBad) != 0;
      uint32_t sr[16];
      if (!bad) {
        ptx::tc_fence_after();
        ptx::tmem_ld16(tmem + lane_base + C::S_COL + kDecTcN * buf, sr);
        ptx::tmem_ld_wait();
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&s_free[buf]);
      const int g = m[1] / p.zgroups, z = m[1] % p.zgroups;
      const long long head0 = static_cast<long long>(m[0]) * p.Hq + g * p.G + z * GT;
      if (!bad) {
        float x[GT];
#pragma unroll
        for (int gh = 0; gh < GT; ++gh)
          x[gh] = t < nt ? __uint_as_float(sr[gh]) * p.scale_log2 : -INFINITY;
        // chunk max per head: warp, then the four warps
        float* rb = red + buf * 64;
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) {
          float mx = x[gh];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          if (lane == 0) rb[warp * 16 + gh] = mx;
        }
        ptx::bar_sync_named(1, 128);
        float alpha[GT];
        bool rescale = false;
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) {
          const float cm = fmaxf(fmaxf(rb[gh], rb[16 + gh]), fmaxf(rb[32 + gh], rb[48 + gh]));
          float m_new = m_run[gh];
          if (!seg_good || cm > m_run[gh] + kDecTcRescale) m_new = fmaxf(m_run[gh], cm);
          alpha[gh] = ptx::ex2(m_run[gh] - m_new);  // 1 when unchanged, 0 at a segment start
          rescale |= seg_good && m_new != m_run[gh];
          m_run[gh] = m_new;
        }
        float pv[GT];
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) {
          pv[gh] = ptx::ex2(x[gh] - m_run[gh]);  // masked tokens: 0
          float sum = pv[gh];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          l_w[gh] = fmaf(l_w[gh], alpha[gh], sum);
        }
        // P buffer ngood & 1 is free once the P.V two good chunks back is done;
        // a rescale rewrites O, so it also waits for the previous P.V
        if (ngood > 1) ok = decode_wait(&pv_done[ngood & 1], ((ngood - 2) >> 1) & 1);
        if (ok && rescale && ngood > 0)
          ok = decode_wait(&pv_done[(ngood - 1) & 1], ((ngood - 1) >> 1) & 1);
        ok = ptx::bar_red_and(1, 128, ok);
        if (!ok) {
          if (tid == 0) decode_error(p, kErrDecodeWait);
          break;
        }
        ptx::tc_fence_after();
        // P[gh][t] as bf16, K-major with the 128-byte swizzle
        {
          const int half = t >> 6, c = t & 63;
#pragma unroll
          for (int gh = 0; gh < GT; ++gh) {
            const uint32_t addr = p_base + (ngood & 1) * C::PBUF + half * C::PHALF + gh * 128 +
                                  ((((c >> 3) ^ (gh & 7))) << 4) + (c & 7) * 2;
            const __nv_bfloat16 bv = __float2bfloat16_rn(pv[gh]);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr),
                         "h"(*reinterpret_cast<const unsigned short*>(&bv))
                         : "memory");
          }
        }
        if (nt < C::CH) {
          // the P.V product reads all 128 V rows: rows past the chunk's tokens
          // (stale cache rows or earlier data) become zero, so 0 * row stays 0
          ok = decode_wait(&full_v[kc % C::NV], (kc / C::NV) & 1);
          ok = ptx::bar_red_and(1, 128, ok);
          if (!ok) {
            if (tid == 0) decode_error(p, kErrDecodeWait);
            break;
          }
          if (t >= nt) {
            uint4* row = reinterpret_cast<uint4*>(sm + C::V_OFF + (kc % C::NV) * C::VSTAGE +
                                                  (t >> 3) * C::ATOM + (t & 7) * 128);
#pragma unroll
            for (int h = 0; h < C::HALVES; ++h)  // columns 64 h .. 64 h + 63
#pragma unroll
              for (int i = 0; i < 8; ++i) row[h * 64 + i] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (rescale) {  // uniform: every thread saw the same maxima
          if constexpr (D == 128) {  // thread = column, one O^T cell per head
            uint32_t ov[16];
            ptx::tmem_ld16(o_addr, ov);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int gh = 0; gh < GT; ++gh)
              ov[gh] = __float_as_uint(__uint_as_float(ov[gh]) * alpha[gh]);
            ptx::tmem_st16(o_addr, ov);
            ptx::tmem_st_wait();
          } else if (warp == 0) {  // lane = query row of O (rows >= GT unused)
            float a = 1.f;
#pragma unroll
            for (int gh = 0; gh < GT; ++gh)
              if (lane == gh) a = alpha[gh];
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
              uint32_t ov[32];
              ptx::tmem_ld32(o_addr + 32 * h, ov);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * a);
              ptx::tmem_st32(o_addr + 32 * h, ov);
            }
            ptx::tmem_st_wait();
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&p_full[ngood & 1]);
        ++ngood;
        seg_good = true;
      }
      if (flags & kStageSegLast) {
        const long long base = head0 * p.nslot + m[5];  // slot of head gh: + gh * nslot
        if (seg_good) {
          ok = decode_wait(&pv_done[(ngood - 1) & 1], ((ngood - 1) >> 1) & 1);
          ok = ptx::bar_red_and(1, 128, ok);
          if (!ok) {
            if (tid == 0) decode_error(p, kErrDecodeWait);
            break;
          }
          ptx::tc_fence_after();
          if constexpr (D == 128) {
            uint32_t ov[16];
            ptx::tmem_ld16(o_addr, ov);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int gh = 0; gh < GT; ++gh)
              p.part_o[(base + gh * p.nslot) * C::D + t] = __uint_as_float(ov[gh]);
          } else if (warp == 0) {
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
              uint32_t ov[32];
              ptx::tmem_ld32(o_addr + 32 * h, ov);
              ptx::tmem_ld_wait();
              if (lane < GT) {
                float4* dst = reinterpret_cast<float4*>(p.part_o + (base + lane * p.nslot) * C::D +
                                                        32 * h);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  dst[i] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                       __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
              }
            }
          }
          if (lane == 0) {
#pragma unroll
            for (int gh = 0; gh < GT; ++gh) lred[warp * 16 + gh] = l_w[gh];
          }
          ptx::bar_sync_named(1, 128);
          if (t < GT) {
            float l = 0.f, mm = 0.f;
#pragma unroll
            for (int gh = 0; gh < GT; ++gh)
              if (gh == t) {
                l = lred[gh] + lred[16 + gh] + lred[32 + gh] + lred[48 + gh];
                mm = m_run[gh];
              }
            float* ml = p.part_ml + (base + t * p.nslot) * 2;
            ml[0] = mm;
            ml[1] = l;
          }
          ptx::bar_sync_named(1, 128);  // lred is free again
        } else if (t < GT) {  // every chunk of the segment was dropped
          float* ml = p.part_ml + (base + t * p.nslot) * 2;
          ml[0] = -INFINITY;
          ml[1] = 0.f;
        }
        if ((flags & kStageItemLast) && t == 0)
          p.slots[static_cast<long long>(m[0]) * p.Hkv * p.zgroups + m[1]] = m[5] + 1;
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) {
          m_run[gh] = -INFINITY;
          l_w[gh] = 0.f;
        }
        seg_good = false;
      }
    }
    ptx::tc_fence_before();
    ptx::bar_arrive_named(2, 160);  // tensor memory may be released
  }
}

}  // namespace tessera
