// Causal grouped-query FlashAttention forward for B200 (sm_100a), CTA-pair form.
//
// Method: FlashAttention forward with online softmax, causal masking and
// grouped-query attention, as named by the Tessera pages (hysenlabs.com
// Tessera review, "The kernel set and its torch fallback"; Tessera README,
// "What's in it" / "Kernels").  This file holds the head-dimension-128,
// fixed-length form built on CTA pairs; attn_fwd_sm100.cuh holds the
// single-CTA form (head dimension 64, packed sequences).
//
// A cluster of two CTAs works on one unit at a time: 256 query rows, 128 per
// CTA, that read the same key/value head (two query heads of a group at the
// same rows when the group size G is even, else two consecutive 128-row
// blocks of one head).  The even CTA's MMA thread issues tcgen05 MMAs with
// cta_group::2 (M = 256): each CTA holds its own 128 query rows, its own rows
// of every accumulator, and HALF of each key/value tile (keys 64r..64r+63 of
// K, columns 64r..64r+63 of V for CTA r), so each K/V byte crosses into
// shared memory once per 256 query rows and each CTA's shared-memory port
// carries half the B-operand reads.
//
// Tensor memory per CTA (512 columns x 128 lanes, fp32 cells):
//   S_b = Q K_j^T    columns [128 b, 128 b + 128), b = j mod 3
//   P_b (bf16 pairs) columns [128 b, 128 b + 64), written over S_b
//   O                columns [384, 512)
// Three S buffers let S(j+1) and S(j+2) be computed while the softmax works on
// S(j): the MMA order per unit is S(0), S(1), S(2), then PV(j), S(j+3) for
// j = 0, 1, ...  tcgen05 MMAs from one thread execute in order, so S(j+3)
// overwrites buffer j mod 3 only after PV(j) has read P(j) from it.
//
// Warp roles (192 threads per CTA):
//   warps 0-3  softmax + epilogue of this CTA's 128 rows (thread r owns row r)
//   warp  4    TMEM allocation (both CTAs) and MMA issue (even CTA, one lane)
//   warp  5    TMA producer: this CTA's Q tile and halves of K/V tiles
//
// Barriers: "full" barriers of the ring and of Q live in the even CTA (both
// CTAs' copies count their bytes there); "empty" barriers, S-ready, PV-done
// and O-ready are signalled to both CTAs by multicast commits; P-ready lives
// in the even CTA and takes one arrival from each of the eight softmax warps.
// The running max is rescaled lazily (O and l keep a stale max until the row
// max grows by more than 2^8, exact because both carry the same max).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace tessera {

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int BM = 128;                  // query rows per CTA
  static constexpr int BN = 128;                  // keys per tile
  static constexpr int SUB_BYTES = 128 * 128;     // [128 rows x 64 bf16] swizzled sub-tile
  static constexpr int TILE_BYTES = 128 * D * 2;  // one [128 x 128] bf16 tile
  static constexpr int HALF_BYTES = TILE_BYTES / 2;  // this CTA's half of a K or V tile
  static constexpr int KSUB_BYTES = 64 * 128;     // [64 keys x 64 bf16] sub-tile of a K half
  static constexpr int NQBUF = 2;                 // Q buffers (the next unit's Q loads early)
  static constexpr int NSTAGE = 8;                // K/V half-tile ring
  static constexpr int NSBUF = 3;                 // S buffers in TMEM
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = Q_OFF + NQBUF * TILE_BYTES;
  static constexpr int OST_OFF = KV_OFF + NSTAGE * HALF_BYTES;  // O staging for the TMA store
  static constexpr int BAR_OFF = OST_OFF + TILE_BYTES;
  // q_full[2] q_empty[2] kv_full[NS] kv_empty[NS] s_full[3] p_full[3] pv_done[2] o_full drain
  static constexpr int NBAR = 2 * NQBUF + 2 * NSTAGE + 2 * NSBUF + 2 + 2;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int O_COL = NSBUF * 128;
  static constexpr int THREADS = 192;
  static constexpr int MMA_WARP = 4;
  static constexpr int TMA_WARP = 5;
  static constexpr int SOFTMAX_BAR = 1;           // named barrier of the 128 softmax threads
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL + D <= 512, "tensor memory budget");
};

// The k-th unit of this CTA pair (snake order over the heaviest-first list;
// both CTAs of a cluster walk the same units), or -1.
__device__ __forceinline__ int pair_unit_of(const FwdParams& p, int k) {
  const int clusters = static_cast<int>(gridDim.x) >> 1;
  const int cid = static_cast<int>(blockIdx.x) >> 1;
  const int c = (k & 1) ? (clusters - 1 - cid) : cid;
  const long long u = static_cast<long long>(k) * clusters + c;
  return u < p.num_units ? static_cast<int>(u) : -1;
}

// wait_bounded on a barrier whose phase completes through arrivals from the
// peer CTA (acquire at cluster scope).
__device__ __forceinline__ bool wait_bounded_cluster(uint64_t* bar, uint32_t parity, uint32_t code,
                                                     unsigned long long launch_id) {
  if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 1023u) == 0) {
      const unsigned long long w = *reinterpret_cast<volatile unsigned long long*>(&g_tessera_err);
      if ((w >> 32) == (launch_id & 0xffffffffull) && (w & 0xffffffffull) != 0) return false;
      if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicExch(&g_tessera_err, ((launch_id & 0xffffffffull) << 32) | code);
        return false;
      }
    }
  }
}

// The MMA sequence of a unit with n key tiles: S(0..min(n,3)-1), then for
// each j: PV(j) followed by S(j+3) when j + 3 < n.  op in [0, 2n): returns
// the key tile and sets is_pv.
__device__ __forceinline__ int pair_op(int op, int n, bool& is_pv) {
  const int head = n < 3 ? n : 3;
  if (op < head) {
    is_pv = false;
    return op;
  }
  const int r = op - head;  // alternates PV(0), S(3), PV(1), S(4), ... until the S run out
  const int tail_s = n - head;  // S(3..n-1)
  if (r < 2 * tail_s) {
    is_pv = (r & 1) == 0;
    return is_pv ? (r >> 1) : (r >> 1) + 3;
  }
  is_pv = true;
  return tail_s + (r - 2 * tail_s);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::THREADS, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + C::NQBUF;
  uint64_t* kv_full = q_empty + C::NQBUF;
  uint64_t* kv_empty = kv_full + C::NSTAGE;
  uint64_t* s_full = kv_empty + C::NSTAGE;
  uint64_t* p_full = s_full + C::NSBUF;
  uint64_t* pv_done = p_full + C::NSBUF;
  uint64_t* o_full = pv_done + 2;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SLOT_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  constexpr uint16_t kBoth = 0x3;

  // ---- set-up ---------------------------------------------------------------
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQBUF; ++i) {
      ptx::mbar_init(&q_full[i], 1);
      ptx::mbar_init(&q_empty[i], 1);
    }
    for (int s = 0; s < C::NSTAGE; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < C::NSBUF; ++b) {
      ptx::mbar_init(&s_full[b], 1);
      ptx::mbar_init(&p_full[b], 8);  // one arrival per softmax warp of both CTAs
    }
    ptx::mbar_init(&pv_done[0], 1);
    ptx::mbar_init(&pv_done[1], 1);
    ptx::mbar_init(o_full, 1);
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == C::TMA_WARP && lane == 0) {
    ptx::prefetch_tensormap(&tm_q);
    ptx::prefetch_tensormap(&tm_kh);
    ptx::prefetch_tensormap(&tm_v);
    ptx::prefetch_tensormap(&tm_o);
  }
  if (warp == C::MMA_WARP) {
    ptx::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the peer's barriers exist before anything signals them
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::TMA_WARP) {
    // ======================= TMA producer (both CTAs) =======================
    // Per unit: this CTA's Q tile, then its halves of the K/V tiles in the
    // MMA order.  Completions are counted on the even CTA's full barriers;
    // the even CTA's producer announces both CTAs' bytes.
    const bool leader = lane == 0;
    const uint64_t keep = ptx::policy_evict_last();
    const uint64_t once = ptx::policy_evict_first();
    uint8_t* sQ = smem + C::Q_OFF;
    uint8_t* sKV = smem + C::KV_OFF;
    int idx = 0;   // ring position
    int ucnt = 0;  // units with work so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = pair_unit_of(p, k);
      if (u < 0) break;
      const Unit w = decode_unit(p, u);
      const int n = w.nmax;
      if (n == 0) continue;
      const int qb = ucnt & 1;
      if (!warp_wait(&q_empty[qb], ((ucnt >> 1) & 1) ^ 1u, kErrWaitQEmpty, p.launch_id)) {
        ok = false;
        break;
      }
      if (leader) {
        // A tile whose rows all lie past T (the second block of a head with
        // an odd number of blocks) is not loaded: its P is zero.
        const bool q_in1 = w.qblk[1] * C::BM < w.T;
        const uint32_t full = ptx::mapa(ptx::smem_u32(&q_full[qb]), 0);
        if (rank == 0) ptx::mbar_arrive_expect_tx(&q_full[qb], (1 + q_in1) * C::TILE_BYTES);
        const int row = (rank ? w.qblk[1] : w.qblk[0]) * C::BM;
        const int plane = w.b * p.Hq + (rank ? w.head[1] : w.head[0]);
        if (rank == 0 || q_in1)
          for (int c = 0; c < 2; ++c)
            ptx::tma_load_3d_pair(ptx::smem_u32(sQ + qb * C::TILE_BYTES + c * C::SUB_BYTES),
                                  &tm_q, full, c * 64, row, plane, once);
      }
      __syncwarp();
      const int kv_plane = w.b * p.Hkv + w.g;
      for (int op = 0; op < 2 * n; ++op, ++idx) {
        bool is_pv;
        const int j = pair_op(op, n, is_pv);
        const int s = idx % C::NSTAGE;
        if (!warp_wait(&kv_empty[s], ((idx / C::NSTAGE) & 1) ^ 1u, kErrWaitKvEmpty, p.launch_id)) {
          ok = false;
          break;
        }
        if (leader) {
          // The odd CTA's K half is not loaded when all its keys lie past T
          // (those keys are masked; the stage's stale contents are never used).
          const bool k_in1 = j * C::BN + 64 < w.T;
          const uint32_t full = ptx::mapa(ptx::smem_u32(&kv_full[s]), 0);
          if (rank == 0)
            ptx::mbar_arrive_expect_tx(&kv_full[s], (is_pv || k_in1 ? 2 : 1) * C::HALF_BYTES);
          const uint32_t dst = ptx::smem_u32(sKV + s * C::HALF_BYTES);
          if (is_pv) {
            // V_j[:, 64 r .. 64 r + 63]: one [128 keys x 64] box
            ptx::tma_load_3d_pair(dst, &tm_v, full, 64 * static_cast<int>(rank), j * C::BN,
                                  kv_plane, keep);
          } else if (rank == 0 || k_in1) {
            // K_j[64 r .. 64 r + 63, :]: two [64 keys x 64] boxes
            for (int c = 0; c < 2; ++c)
              ptx::tma_load_3d_pair(dst + c * C::KSUB_BYTES, &tm_kh, full, c * 64,
                                    j * C::BN + 64 * static_cast<int>(rank), kv_plane, keep);
          }
        }
        __syncwarp();
      }
      if (ok) ++ucnt;
    }
    (void)ok;
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issue (even CTA) ===========================
    if (rank == 0) {
      const bool leader = lane == 0;
      constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(256, C::BN, false, false);
      constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(256, C::D, false, true);
      constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);  // SBO 1 KB, 128-B swizzle
      const uint32_t q_addr = ptx::smem_u32(smem + C::Q_OFF);
      const uint32_t kv_addr = ptx::smem_u32(smem + C::KV_OFF);
      int idx = 0;   // ring position
      int ucnt = 0;  // units with work so far
      int sidx = 0;  // key tiles so far (S buffer / P / PV numbering)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = pair_unit_of(p, k);
        if (u < 0) break;
        const Unit w = decode_unit(p, u);
        const int n = w.nmax;
        if (n == 0) continue;
        const int qb = ucnt & 1;
        if (!warp_wait(&q_full[qb], (ucnt >> 1) & 1, kErrWaitQ, p.launch_id)) break;
        for (int op = 0; op < 2 * n; ++op, ++idx) {
          bool is_pv;
          const int j = pair_op(op, n, is_pv);
          const int e = sidx + j;  // global tile number
          const int b = e % C::NSBUF;
          if (is_pv) {
            ok = wait_bounded_cluster(&p_full[b], (e / C::NSBUF) & 1, kErrWaitPFull, p.launch_id);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          const int s = idx % C::NSTAGE;
          if (!warp_wait(&kv_full[s], (idx / C::NSTAGE) & 1, kErrWaitKvFull, p.launch_id)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          if (leader) {
            const uint32_t stage = kv_addr + s * C::HALF_BYTES;
            if (is_pv) {
              // O += P_b V_j: A = P (TMEM), B = this CTA pair's V halves (MN-major);
              // K step kk = 16 keys = 2 KB of the V half, 8 TMEM columns of P
              const uint32_t vb_lo = ptx::sdesc_sw128_lo(stage, C::SUB_BYTES);
              const uint32_t pa = tmem + 128 * b;
              ptx::mma_ts_pair(tmem + C::O_COL, pa, vb_lo, kDescHi, kIdescO, j > 0 ? 1u : 0u);
#pragma unroll
              for (int kk = 1; kk < C::BN / 16; ++kk)
                ptx::mma_ts_pair(tmem + C::O_COL, pa + kk * 8, vb_lo + kk * (2048 >> 4), kDescHi,
                                 kIdescO, 1u);
              ptx::tc_commit_pair(&kv_empty[s], kBoth);
              ptx::tc_commit_pair(&pv_done[e & 1], kBoth);
              if (j == n - 1) ptx::tc_commit_pair(o_full, kBoth);
            } else {
              // S_b = Q K_j^T: A = Q (K-major), B = the K halves (K-major); K step
              // kk: +32 B, or the next sub-tile (16 KB for Q, 8 KB for a K half)
              const uint32_t qa_lo = ptx::sdesc_sw128_lo(q_addr + qb * C::TILE_BYTES, 16);
              const uint32_t kb_lo = ptx::sdesc_sw128_lo(stage, 16);
              const uint32_t sd = tmem + 128 * b;
              ptx::mma_ss_pair<0>(sd, qa_lo, kDescHi, kb_lo, kDescHi, kIdescS);
#pragma unroll
              for (int kk = 1; kk < C::D / 16; ++kk) {
                const uint32_t sa = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
                const uint32_t sb = (kk >> 2) * (C::KSUB_BYTES >> 4) + (kk & 3) * 2;
                ptx::mma_ss_pair<1>(sd, qa_lo + sa, kDescHi, kb_lo + sb, kDescHi, kIdescS);
              }
              ptx::tc_commit_pair(&kv_empty[s], kBoth);
              ptx::tc_commit_pair(&s_full[b], kBoth);
              if (j == n - 1) ptx::tc_commit_pair(&q_empty[qb], kBoth);
            }
          }
          __syncwarp();
        }
        if (!ok) break;
        sidx += n;
        ++ucnt;
      }
      // Every MMA issued must finish before tensor memory is released.
      if (leader) ptx::tc_commit_pair(drain, 0x1);
      __syncwarp();
      warp_wait(drain, 0, kErrWaitDrain, p.launch_id);
    }
  } else {
    // ======================= softmax + epilogue (both CTAs) =================
    const int t = static_cast<int>(rank);  // this CTA's tile of the unit
    const int row = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::O_COL;
    const float sl2 = p.scale_log2;
    const uint32_t ost = ptx::smem_u32(smem + C::OST_OFF);
    int sidx = 0;  // key tiles so far
    int ocnt = 0;  // units so far (o_full phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = pair_unit_of(p, k);
      if (u < 0) break;
      const Unit w = decode_unit(p, u);
      const int n = w.nmax;
      if (n == 0) continue;
      // this CTA's tile of the unit (selects keep the Unit in registers)
      const int n_t = t ? w.ntile[1] : w.ntile[0];
      const int qblk = t ? w.qblk[1] : w.qblk[0];
      const int head = t ? w.head[1] : w.head[0];
      const int q_row = qblk * C::BM + row;
      float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale)
      float l = 0.f;        // running sum of 2^(x - m)
      float lb = 0.f;       // running sum of the bf16-rounded 2^(x - m) that P.V applies
      for (int j = 0; j < n; ++j) {
        const int e = sidx + j;
        const int b = e % C::NSBUF;
        if (!warp_wait(&s_full[b], (e / C::NSBUF) & 1, kErrWaitSFull, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + 128 * b;
        uint32_t pk[2][32];
        bool rescale = false;
        float alpha = 1.f;
        if (j < n_t) {
          uint32_t sr[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) ptx::tmem_ld32(s_addr + 32 * c, sr[c]);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) ptx::reg_fence(sr[c]);
          float sv[128];
#pragma unroll
          for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);
          const int kv0 = j * C::BN;
          const bool edge =
              p.causal ? (kv0 + C::BN - 1 > q_row - row) : (kv0 + C::BN > w.T);
          const int lim = p.causal ? min(q_row, w.T - 1) : w.T - 1;  // last visible key
          float applied;
          const float rowsum =
              edge ? softmax_row_tile<true>(sv, pk, m, alpha, rescale, sl2, kv0, lim, applied)
                   : softmax_row_tile<false>(sv, pk, m, alpha, rescale, sl2, kv0, lim, applied);
          l = l * alpha + rowsum;
          lb = lb * alpha + applied;
        } else {
          // keys past this tile's causal extent (the pair's other tile needs
          // them): P = 0
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[0][i] = pk[1][i] = 0u;
        }
        ptx::tmem_st32(s_addr + 0, pk[0]);
        ptx::tmem_st32(s_addr + 32, pk[1]);
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O *= alpha once PV(j-1) is complete (PV(j) waits for this P)
          if (!warp_wait(&pv_done[(e - 1) & 1], ((e - 1) >> 1) & 1, kErrWaitOFull, p.launch_id)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int c = 0; c < C::D / 32; ++c) {
            uint32_t ov[32];
            ptx::tmem_ld32(o_addr + 32 * c, ov);
            ptx::tmem_ld_wait();
            ptx::reg_fence(ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            ptx::tmem_st32(o_addr + 32 * c, ov);
          }
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(&p_full[b]), 0));
      }
      sidx += n;

      // ---- epilogue: O / l -> bf16 through shared memory, one TMA store ------
      // Every softmax warp reaches each named barrier of a unit exactly once,
      // even after a wait gave up (a warp that gave up votes false), so no
      // warp can be left waiting at a barrier the others skipped.
      if (ok) ok = warp_wait(o_full, ocnt & 1, kErrWaitOFull, p.launch_id);
      ++ocnt;
      // the previous unit's store must have read the staging buffer
      if (threadIdx.x == 0) ptx::bulk_wait_group_read0();
      ok = ptx::bar_red_and(C::SOFTMAX_BAR, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const float inv_l = (lb > 0.f) ? 1.f / lb : 0.f;
#pragma unroll
      for (int c = 0; c < C::D / 32; ++c) {
        uint32_t ov[32];
        ptx::tmem_ld32(o_addr + 32 * c, ov);
        ptx::tmem_ld_wait();
        ptx::reg_fence(ov);
        uint32_t pkd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pkd[i] = ptx::pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l,
                                    __uint_as_float(ov[2 * i + 1]) * inv_l);
        // columns 32c..32c+31 = 16-byte chunks 4(c&1)..4(c&1)+3 of sub-tile c>>1,
        // stored at the 128-byte swizzle's position for this row
        const uint32_t sub = ost + (c >> 1) * C::SUB_BYTES + row * 128;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint32_t chunk = static_cast<uint32_t>(4 * (c & 1) + v4) ^ (row & 7);
          ptx::st_shared_v4(sub + chunk * 16, pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2],
                            pkd[4 * v4 + 3]);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::bar_sync_named(C::SOFTMAX_BAR, 128);
      const int plane = w.b * p.Hq + head;
      if (threadIdx.x == 0 && qblk * C::BM < w.T) {
        // rows past T are clipped by the tensor map
        for (int c = 0; c < 2; ++c)
          ptx::tma_store_3d(&tm_o, ost + c * C::SUB_BYTES, c * 64, qblk * C::BM, plane);
        ptx::bulk_commit_group();
      }
      if (q_row < w.T && p.lse != nullptr)
        p.lse[static_cast<int64_t>(plane) * p.T + q_row] =
            (l > 0.f) ? (m + ptx::lg2(l)) * 0.69314718055994530942f : -INFINITY;
      // O has been read; the next unit's first P arrival (after this fence)
      // is what lets the MMA warp overwrite it.
      ptx::tc_fence_before();
    }
    if (threadIdx.x == 0) ptx::bulk_wait_group0();
  }

  // ---- teardown -------------------------------------------------------------
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the even CTA's MMAs no longer read this CTA's memory
  if (warp == C::MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace tessera
