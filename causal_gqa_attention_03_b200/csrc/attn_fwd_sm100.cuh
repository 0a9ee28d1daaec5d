// Causal grouped-query FlashAttention forward for B200 (sm_100a).
//
// Method: FlashAttention forward with online softmax, causal masking and
// grouped-query attention, as named by the Tessera pages (hysenlabs.com
// Tessera review, "The kernel set and its torch fallback"; Tessera README,
// "What's in it" / "Kernels").  The tile design below is this library's own,
// built for sm_100a: TMA + mbarrier pipeline, tcgen05 MMAs accumulating in
// tensor memory, warp-specialised roles, persistent CTAs.
//
// Work unit: two 128-row query tiles that read the same key/value head.  When
// the group size G is even the two tiles are two query heads of one group at
// the same rows (so each K/V tile fetched into shared memory feeds both);
// otherwise they are two consecutive 128-row blocks of one head.  Units are
// numbered heaviest-first (longest causal extent) and dealt to one CTA per SM
// in snake order, so the causal triangle balances.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3   softmax + epilogue for query tile 0 (thread r owns row r)
//   warps 4-7   softmax + epilogue for query tile 1
//   warp  8     MMA issue (one lane) and TMEM allocation
//   warp  9     TMA producer (one lane)
//   warps 10-11 idle (they complete the third warpgroup for setmaxnreg)
//
// Tensor memory (512 columns x 128 lanes, fp32 cells):
//   S_t = Q_t K_j^T  columns [128 t, 128 t + 128)      (t = 0, 1)
//   P_t (bf16 pairs) columns [128 t, 128 t + 64), written over S_t
//   O_t             columns [256 + D t, 256 + D t + D)
//
// Per key tile j and query tile t the MMA warp issues PV_t(j-1) then S_t(j);
// tcgen05 MMAs from one thread execute in order, so S_t(j) cannot overwrite
// P_t(j-1) before PV_t(j-1) has read it.  The softmax of tile t overlaps the
// MMAs of the other tile.  Across units the same order holds: a unit's first
// S_t follows the previous unit's last PV_t, and its first PV_t (which
// overwrites O_t) waits for P_t, which the softmax writes only after its
// epilogue has read O_t.  The running max is rescaled lazily: O and l keep a
// stale max until the row max grows by more than 2^64, which is exact because
// both carry the same max.  Weights then reach 2^64, so the fp32 O and l stay
// finite while |V| * T < 2^63 (|V| < 2^49 at T = 16384).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "exp2_fma.cuh"
#include "sm100_ptx.cuh"

namespace tessera {

// Device error word: high 32 bits = launch id, low 32 bits = code of the wait
// that gave up.  Nonzero only after a bounded wait expired.
__device__ unsigned long long g_tessera_err = 0ull;

enum WaitCode : uint32_t {
  kErrWaitQ = 1,
  kErrWaitKvEmpty = 2,
  kErrWaitKvFull = 3,
  kErrWaitSFull = 4,
  kErrWaitPFull = 5,
  kErrWaitOFull = 6,
  kErrWaitDrain = 7,
  kErrWaitQEmpty = 8,
  kErrSelfTest = 9,  // the deliberate timeout of attn_selftest_timeout_kernel
  kErrVarlenInput = 10,  // a packed sequence's bounds out of range (that sequence is skipped)
};

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait
constexpr float kRescaleThreshold = 64.0f;         // log2 units: rescale when the max grows > 2^64
// Of the 128 exponentials per row and key tile, this many (the last columns)
// run on the FMA pipe (exp2_fma2) instead of MUFU, in tiles without masking.
// Measured on B200 at the 1 kW power cap: 0 is fastest for long sequences
// (each emulated exp costs ~8 FMA-pipe instructions, which lowers the
// power-capped clock more than the MUFU work it saves), 32 is marginally
// faster for T = 4096.
constexpr int kEmuCols = 0;

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BM = 128;                  // query rows per tile
  static constexpr int BN = 128;                  // keys per tile
  static constexpr int NQ = 2;                    // query tiles per unit
  static constexpr int SUB = D / 64;              // 128-byte-wide column sub-tiles per tile
  static constexpr int SUB_BYTES = 128 * 128;     // one [128 rows x 64 bf16] sub-tile
  static constexpr int TILE_BYTES = 128 * D * 2;  // one [128 x D] bf16 tile
  static constexpr int NSTAGE = (D == 128) ? 5 : 8;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = NQ * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSTAGE * TILE_BYTES;
  // q_full, q_empty, kv_full[NSTAGE], kv_empty[NSTAGE], s_full[NQ], p_full[NQ],
  // o_full[NQ], drain
  static constexpr int NBAR = 2 + 2 * NSTAGE + 3 * NQ + 1;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int S_COL = 0;
  static constexpr int O_COL = 256;
  static constexpr int THREADS = 384;             // three warpgroups
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  // Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512);
  // the MMA/TMA warpgroup gives registers back, the softmax warpgroups take
  // them: 2 x 128 x 200 + 128 x 96 = 63488 <= 64512.
  static constexpr int REGS_SOFTMAX = 200;
  static constexpr int REGS_OTHER = 96;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL + NQ * D <= 512, "tensor memory budget");
  static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_OTHER <= THREADS * 168, "register split");
};

struct FwdParams {
  int B, Hq, Hkv, T, G;
  int causal;
  float scale_log2;          // scale * log2(e)
  int nqb;                   // ceil(T / 128)
  int pair_heads;            // 1: tiles are heads (2p, 2p+1) of a group; 0: q-blocks (2p, 2p+1)
  int units_per_step;        // units sharing one position in the heaviest-first order
  int r_group;               // positions r of a step walked together (units_per_step: all)
  int num_units;
  __nv_bfloat16* o;
  float* lse;
  unsigned long long launch_id;
  // Packed sequences: cu_seqlens[b] .. cu_seqlens[b+1] are sequence b's rows
  // of q [total, Hq, d], k/v [total, Hkv, d], o [total, Hq, d], lse [Hq, total];
  // T is then the longest length.  Null: fixed length T, layouts [B, H, T, d].
  const int* cu_seqlens;
  int total;
};

// A work unit: batch b, key/value head g, the two tiles' query heads and
// 128-row blocks, and how many key tiles each visits (0: tile absent).  T is
// the sequence's length and row0 its first row in the packed layout (0 for
// fixed-length batches).
struct Unit {
  int b, g;
  int head[2], qblk[2], ntile[2];
  int nmax;
  int T, row0;
};

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  Unit w;
  int step, r;
  if (p.r_group < p.units_per_step) {
    // Grouped: the units of positions r in [0, r_group), heaviest first, then
    // those of [r_group, 2 r_group), ...  Consecutive positions share a
    // (batch, key/value head) slice, so the CTAs work on one group's keys and
    // values at a time and those stay in L2: one sequence of a packed batch,
    // or as many slices as half of L2 holds when the whole K/V does not fit.
    const int nsteps = p.num_units / p.units_per_step;
    const int per_group = p.r_group * nsteps;
    const int gi = u / per_group;
    const int rest = u % per_group;
    const int rg = min(p.r_group, p.units_per_step - gi * p.r_group);
    step = rest / rg;
    r = gi * p.r_group + rest % rg;
  } else {
    step = u / p.units_per_step;
    r = u % p.units_per_step;
  }
  if (p.pair_heads) {
    const int half = p.G >> 1;
    const int hp = r % half;
    const int bg = r / half;
    w.b = bg / p.Hkv;
    w.g = bg % p.Hkv;
    w.head[0] = w.g * p.G + 2 * hp;
    w.head[1] = w.head[0] + 1;
    w.qblk[0] = w.qblk[1] = p.nqb - 1 - step;
  } else {
    const int npairs = (p.nqb + 1) >> 1;
    const int pr = npairs - 1 - step;
    w.b = r / p.Hq;
    w.head[0] = w.head[1] = r % p.Hq;
    w.g = w.head[0] / p.G;
    w.qblk[0] = 2 * pr;
    w.qblk[1] = 2 * pr + 1;
  }
  w.T = p.T;
  w.row0 = 0;
  if (p.cu_seqlens != nullptr) {
    const int start = p.cu_seqlens[w.b], end = p.cu_seqlens[w.b + 1];
    if (start < 0 || end < start || end - start > p.T || end > p.total) {
      // skip the sequence; recorded under another launch id, so that the
      // other units' bounded waits carry on
      atomicCAS(&g_tessera_err, 0ull,
                (((p.launch_id ^ 0x80000000ull) & 0xffffffffull) << 32) | kErrVarlenInput);
      w.T = 0;
    } else {
      w.T = end - start;
      w.row0 = start;
    }
  }
  const int nqb = (w.T + 127) / 128;
#pragma unroll
  for (int t = 0; t < 2; ++t)
    w.ntile[t] = (w.qblk[t] >= nqb) ? 0 : (p.causal ? min(w.qblk[t] + 1, nqb) : nqb);
  w.nmax = max(w.ntile[0], w.ntile[1]);
  return w;
}

// The k-th unit of this CTA (snake order over the heaviest-first list), or -1.
__device__ __forceinline__ int unit_of(const FwdParams& p, int k) {
  const int c = (k & 1) ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                        : static_cast<int>(blockIdx.x);
  const long long u = static_cast<long long>(k) * gridDim.x + c;
  return u < p.num_units ? static_cast<int>(u) : -1;
}

// Wait for the phase of `parity` on `bar`, giving up after limit_ns or as
// soon as another CTA of the same launch has given up.  Returns false on give-up.
// A phase that has already completed is seen by the non-blocking test (the
// blocking try_wait costs a few hundred cycles even then).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, uint32_t code,
                                             unsigned long long launch_id,
                                             uint64_t limit_ns = kWaitLimitNs) {
  if (ptx::mbar_test_wait(bar, parity)) return true;
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 0) {
      const unsigned long long w = *reinterpret_cast<volatile unsigned long long*>(&g_tessera_err);
      if ((w >> 32) == (launch_id & 0xffffffffull) && (w & 0xffffffffull) != 0) return false;
      if (ptx::globaltimer_ns() - t0 > limit_ns) {
        atomicExch(&g_tessera_err, ((launch_id & 0xffffffffull) << 32) | code);
        return false;
      }
    }
  }
}

// Diagnostic: one warp waits, through wait_bounded, on an mbarrier that
// nothing arrives at, so the wait gives up after limit_ns and records
// kErrSelfTest in the error word.  It exercises the path every wait of the
// attention kernel takes when it gives up, without faulting or hanging.
__global__ void __launch_bounds__(32, 1)
    attn_selftest_timeout_kernel(unsigned long long launch_id, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) wait_bounded(&bar, 0, kErrSelfTest, launch_id, limit_ns);
  __syncwarp();
}

// All lanes wait; the warp proceeds only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t code,
                                          unsigned long long launch_id) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, code, launch_id));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Online-softmax step for one row (this thread) and one 128-key tile.
// s: the row's 128 raw scores.  Masked keys (kv0 + c > lim) become -inf when
// kMasked.  Updates the running (possibly stale) max m in scaled log2 units,
// sets alpha = 2^(m_old - m_new) (1 when m is kept) and rescale, writes P as
// bf16 pairs into pk, and returns the row sum of the fp32 p (for the LSE)
// and, in applied, the row sum of the bf16-rounded p that the P.V product
// applies (O is normalised by it, so O stays an exact convex combination of
// V rows whatever the rounding of the dominant weights).
template <bool kMasked>
__device__ __forceinline__ float softmax_row_tile(float (&s)[128], uint32_t (&pk)[2][32], float& m,
                                                  float& alpha, bool& rescale, float sl2, int kv0,
                                                  int lim, float& applied) {
  if (kMasked) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (kv0 + c > lim) s[c] = -INFINITY;
  }
  // row max: eight independent chains of 3-input max
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = s[k];
#pragma unroll
  for (int i = 0; i < 60; ++i) mx[i & 7] = max3f(mx[i & 7], s[8 + 2 * i], s[9 + 2 * i]);
  const float mrow = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]),
                           fmaxf(mx[6], mx[7]));
  const float m_tile = mrow * sl2;
  alpha = 1.f;
  rescale = m_tile > m + kRescaleThreshold;  // always true on the first tile (m = -inf)
  if (rescale) {
    alpha = ptx::ex2(m - m_tile);
    m = m_tile;
  }
  const float neg_m = (m == -INFINITY) ? 0.f : -m;
  const float2 sl2_2 = make_float2(sl2, sl2);
  const float2 nm_2 = make_float2(neg_m, neg_m);
  float2 acc[4], accb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = accb[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sl2_2, nm_2);
    float2 pv;
    if (!kMasked && 2 * c >= 128 - kEmuCols) {
      pv = exp2_fma2(x);
    } else {
      pv.x = ptx::ex2(x.x);
      pv.y = ptx::ex2(x.y);
    }
    acc[c & 3] = __fadd2_rn(acc[c & 3], pv);
    const uint32_t packed = ptx::pack_bf16x2(pv.x, pv.y);
    pk[c >> 5][c & 31] = packed;
    accb[c & 3] = __fadd2_rn(accb[c & 3], ptx::bf16x2_to_float2(packed));
  }
  const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  const float2 ab = __fadd2_rn(__fadd2_rn(accb[0], accb[1]), __fadd2_rn(accb[2], accb[3]));
  applied = ab.x + ab.y;
  return a.x + a.y;
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sKV = smem + C::KV_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + C::NSTAGE;
  uint64_t* s_full = kv_empty + C::NSTAGE;
  uint64_t* p_full = s_full + C::NQ;
  uint64_t* o_full = p_full + C::NQ;
  uint64_t* drain = o_full + C::NQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SLOT_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up ---------------------------------------------------------------
  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_empty, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < C::NQ; ++t) {
      ptx::mbar_init(&s_full[t], 1);
      ptx::mbar_init(&p_full[t], 4);  // one arrival per softmax warp
      ptx::mbar_init(&o_full[t], 1);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == C::TMA_WARP && lane == 0) {
    ptx::prefetch_tensormap(&tm_q);
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
  }
  if (warp == C::MMA_WARP) {
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    // ---- third warpgroup: gives registers back, then TMA and MMA issue ------
    ptx::setmaxnreg_dec<C::REGS_OTHER>();
    if (warp == C::TMA_WARP) {
      // ======================= TMA producer =================================
      // Per unit: Q tiles (once the previous unit's S products are done with
      // the Q buffer), then K_0, V_0, K_1, V_1, ... into the ring.  The whole
      // warp runs the loop and waits (a converged warp resumes from an
      // mbarrier wait sooner than a single lane does); lane 0 issues.
      const bool leader = lane == 0;
      // K/V tiles are re-read by the other units of the same key/value head:
      // keep them in L2; Q is read once.
      const uint64_t keep = ptx::policy_evict_last();
      const uint64_t once = ptx::policy_evict_first();
      int idx = 0;  // K/V tiles loaded so far (ring position)
      int kq = 0;   // units with work so far (Q buffer phases)
      const bool packed = p.cu_seqlens != nullptr;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(p, k);
        if (u < 0) break;
        const Unit w = decode_unit(p, u);
        if (w.nmax == 0) continue;  // past the end of a short packed sequence
        // Q of this unit, once the previous unit's S products no longer read
        // the Q buffer.  Fixed length: (row, plane b*H + h); packed: the map
        // is [total][H][d], coordinates (head, row).
        auto load_q = [&]() -> bool {
          if (!warp_wait(q_empty, (kq & 1) ^ 1u, kErrWaitQEmpty, p.launch_id)) return false;
          if (leader) {
            ptx::mbar_arrive_expect_tx(q_full,
                                       ((w.ntile[0] > 0) + (w.ntile[1] > 0)) * C::TILE_BYTES);
            for (int t = 0; t < C::NQ; ++t) {
              if (w.ntile[t] == 0) continue;
              const int row = w.row0 + w.qblk[t] * C::BM;
              const int y = packed ? w.head[t] : row;
              const int z = packed ? row : w.b * p.Hq + w.head[t];
              for (int c = 0; c < C::SUB; ++c)
                ptx::tma_load_3d_hint(sQ + t * C::TILE_BYTES + c * C::SUB_BYTES, &tm_q, q_full,
                                      c * 64, y, z, once);
            }
          }
          __syncwarp();
          return true;
        };
        const int kv_plane = packed ? w.g : w.b * p.Hkv + w.g;
        // K_0 and V_0 go first: they do not depend on the Q buffer
        const int q_at = min(2, 2 * w.nmax);
        for (int i = 0; i < 2 * w.nmax; ++i, ++idx) {  // K_0, V_0, K_1, V_1, ...
          if (i == q_at && !load_q()) {
            ok = false;
            break;
          }
          const int s = idx % C::NSTAGE;
          if (!warp_wait(&kv_empty[s], ((idx / C::NSTAGE) & 1) ^ 1u, kErrWaitKvEmpty,
                         p.launch_id)) {
            ok = false;
            break;
          }
          if (leader) {
            ptx::mbar_arrive_expect_tx(&kv_full[s], C::TILE_BYTES);
            const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
            const int row = w.row0 + (i >> 1) * C::BN;
            for (int c = 0; c < C::SUB; ++c)
              ptx::tma_load_3d_hint(sKV + s * C::TILE_BYTES + c * C::SUB_BYTES, map, &kv_full[s],
                                    c * 64, packed ? kv_plane : row, packed ? row : kv_plane,
                                    keep);
          }
          __syncwarp();
        }
        if (ok && q_at == 2 * w.nmax && !load_q()) ok = false;
        if (ok) ++kq;
      }
      if (!ok) {
        // Gave up: let the copies already in flight land before the CTA exits.
        if (kq > 0) warp_wait(q_full, (kq - 1) & 1, kErrWaitQ, p.launch_id);
        for (int i = max(0, idx - C::NSTAGE); i < idx; ++i)
          warp_wait(&kv_full[i % C::NSTAGE], (i / C::NSTAGE) & 1, kErrWaitKvFull, p.launch_id);
      }
    } else if (warp == C::MMA_WARP) {
      // ======================= MMA issue ====================================
      // The whole warp runs the loop and waits; lane 0 issues the MMAs and
      // the commits (a commit tracks the MMAs of the thread that issues it).
      const bool leader = lane == 0;
      constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);  // SBO 1 KB, 128-B swizzle
      const uint32_t q_addr = ptx::smem_u32(sQ);
      const uint32_t kv_addr = ptx::smem_u32(sKV);
      int base = 0;           // ring position of the unit's K_0
      int pcnt[2] = {0, 0};   // P tiles consumed per query tile (p_full phases)
      bool ok = true;
      int kq = 0;  // units with work so far (Q buffer phases)
      for (int k = 0; ok; ++k) {
        const int u = unit_of(p, k);
        if (u < 0) break;
        const Unit w = decode_unit(p, u);
        if (w.nmax == 0) continue;  // past the end of a short packed sequence
        if (!warp_wait(q_full, kq & 1, kErrWaitQ, p.launch_id)) break;
        ++kq;
        for (int j = 0; ok && j <= w.nmax; ++j) {
          const int kidx = base + 2 * j, vidx = base + 2 * j - 1;
          if (j < w.nmax)
            ok = warp_wait(&kv_full[kidx % C::NSTAGE], (kidx / C::NSTAGE) & 1, kErrWaitKvFull,
                           p.launch_id);
          if (ok && j > 0)
            ok = warp_wait(&kv_full[vidx % C::NSTAGE], (vidx / C::NSTAGE) & 1, kErrWaitKvFull,
                           p.launch_id);
          if (!ok) break;
          ptx::tc_fence_after();
          for (int t = 0; t < C::NQ && ok; ++t) {
            if (j >= 1 && j <= w.ntile[t]) {
              // O_t += P_t(j-1) V_{j-1}; A = P from TMEM, B = V (MN-major in smem)
              ok = warp_wait(&p_full[t], pcnt[t] & 1, kErrWaitPFull, p.launch_id);
              if (!ok) break;
              ++pcnt[t];
              ptx::tc_fence_after();
              if (leader) {
                // B descriptor low word of the V tile; K step kk is 16 keys = 2 KB further
                const uint32_t vb_lo =
                    ptx::sdesc_sw128_lo(kv_addr + (vidx % C::NSTAGE) * C::TILE_BYTES, C::SUB_BYTES);
                const uint32_t pa = tmem + C::S_COL + 128 * t;
                ptx::mma_ts_lohi_rt(tmem + C::O_COL + D * t, pa, vb_lo, kDescHi, kIdescO,
                                    j > 1 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < C::BN / 16; ++kk)
                  ptx::mma_ts_lohi<1>(tmem + C::O_COL + D * t, pa + kk * 8,
                                      vb_lo + kk * (2048 >> 4), kDescHi, kIdescO);
                if (j == w.ntile[t]) ptx::tc_commit(&o_full[t]);
              }
              __syncwarp();
            }
            if (j < w.ntile[t]) {
              if (leader) {
                // S_t = Q_t K_j^T; both operands K-major in smem.  A and B
                // descriptor low words; K step kk: +32 B, or the next 16 KB sub-tile
                const uint32_t qa_lo = ptx::sdesc_sw128_lo(q_addr + t * C::TILE_BYTES, 16);
                const uint32_t kb_lo =
                    ptx::sdesc_sw128_lo(kv_addr + (kidx % C::NSTAGE) * C::TILE_BYTES, 16);
                const uint32_t sd = tmem + C::S_COL + 128 * t;
                ptx::mma_ss_lohi<0>(sd, qa_lo, kDescHi, kb_lo, kDescHi, kIdescS);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk) {
                  const uint32_t st = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
                  ptx::mma_ss_lohi<1>(sd, qa_lo + st, kDescHi, kb_lo + st, kDescHi, kIdescS);
                }
                ptx::tc_commit(&s_full[t]);
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          if (leader) {
            if (j < w.nmax) ptx::tc_commit(&kv_empty[kidx % C::NSTAGE]);
            if (j > 0) ptx::tc_commit(&kv_empty[vidx % C::NSTAGE]);
            // the unit's last S products: the Q buffer is free once they complete
            if (j == w.nmax - 1) ptx::tc_commit(q_empty);
          }
          __syncwarp();
        }
        base += 2 * w.nmax;
      }
      // Every MMA issued must finish before tensor memory is released.
      if (leader) ptx::tc_commit(drain);
      __syncwarp();
      warp_wait(drain, 0, kErrWaitDrain, p.launch_id);
    }
  } else {
    ptx::setmaxnreg_inc<C::REGS_SOFTMAX>();
    // ======================= softmax + epilogue =============================
    const int t = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + C::S_COL + 128 * t;
    const uint32_t o_addr = tmem + lane_base + C::O_COL + D * t;
    const float sl2 = p.scale_log2;
    int scnt = 0;  // S tiles of this query tile seen so far (s_full phases)
    int ocnt = 0;  // units of this query tile finished so far (o_full phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_of(p, k);
      if (u < 0) break;
      const Unit w = decode_unit(p, u);
      const int n_t = w.ntile[t];
      if (n_t == 0) continue;
      const int q_row = w.qblk[t] * C::BM + row;
      float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale)
      float l = 0.f;        // running sum of 2^(x - m)
      float lb = 0.f;       // running sum of the bf16-rounded 2^(x - m) that P.V applies
      for (int j = 0; j < n_t; ++j) {
        if (!warp_wait(&s_full[t], scnt & 1, kErrWaitSFull, p.launch_id)) {
          ok = false;
          break;
        }
        ++scnt;
        ptx::tc_fence_after();
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
        const bool edge = p.causal ? (kv0 + C::BN - 1 > q_row - row) : (kv0 + C::BN > w.T);
        const int lim = p.causal ? min(q_row, w.T - 1) : w.T - 1;  // last visible key
        float alpha;
        bool rescale;
        uint32_t pk[2][32];
        float applied;
        const float rowsum =
            edge ? softmax_row_tile<true>(sv, pk, m, alpha, rescale, sl2, kv0, lim, applied)
                 : softmax_row_tile<false>(sv, pk, m, alpha, rescale, sl2, kv0, lim, applied);
        l = l * alpha + rowsum;
        lb = lb * alpha + applied;
        ptx::tmem_st32(s_addr + 0, pk[0]);
        ptx::tmem_st32(s_addr + 32, pk[1]);
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O_t *= alpha (PV_t(j-1) is complete: S_t(j) was committed after it)
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
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
        if (lane == 0) ptx::mbar_arrive(&p_full[t]);
      }
      if (!ok) break;

      // ---- epilogue: O / l -> bf16, LSE -----------------------------------------
      if (!warp_wait(&o_full[t], ocnt & 1, kErrWaitOFull, p.launch_id)) break;
      ++ocnt;
      ptx::tc_fence_after();
      const float inv_l = (lb > 0.f) ? 1.f / lb : 0.f;
      const bool store = q_row < w.T;
      // O and LSE element offsets of this row: [B,Hq,T,d] / [B,Hq,T], or packed
      // [total,Hq,d] / [Hq,total]
      int64_t orow, lrow;
      if (p.cu_seqlens != nullptr) {
        const int64_t tok = static_cast<int64_t>(w.row0) + q_row;
        orow = tok * p.Hq + w.head[t];
        lrow = static_cast<int64_t>(w.head[t]) * p.total + tok;
      } else {
        orow = (static_cast<int64_t>(w.b) * p.Hq + w.head[t]) * p.T + q_row;
        lrow = orow;
      }
      // The row as D/8 pieces of 16 bytes, then stored by lane pairs: lanes
      // 2m and 2m+1 swap one piece per step (shfl.xor 1), so every warp store
      // writes 32 contiguous bytes of each of 16 rows -- whole 32-byte
      // sectors, 16 per 512-byte request.
      uint32_t packed[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        ptx::tmem_ld32(o_addr + 32 * c, ov);
        ptx::tmem_ld_wait();
        ptx::reg_fence(ov);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[16 * c + i] = ptx::pack_bf16x2(__uint_as_float(ov[2 * i]) * inv_l,
                                               __uint_as_float(ov[2 * i + 1]) * inv_l);
      }
      const bool odd = lane & 1;
      __nv_bfloat16* const dst = p.o + orow * D;
      const unsigned long long dst_bits = reinterpret_cast<unsigned long long>(dst);
      uint4* const row_even =
          reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, dst_bits, lane & ~1));
      uint4* const row_odd =
          reinterpret_cast<uint4*>(__shfl_sync(0xffffffffu, dst_bits, lane | 1));
      const bool st_even = __shfl_sync(0xffffffffu, store, lane & ~1);
      const bool st_odd = __shfl_sync(0xffffffffu, store, lane | 1);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        // pieces 2k (even lane's) and 2k+1 (odd lane's) of both rows
        uint32_t send[4], recv[4], v1[4], v2[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          send[w] = odd ? packed[8 * k + w] : packed[8 * k + 4 + w];
          recv[w] = __shfl_xor_sync(0xffffffffu, send[w], 1);
          v1[w] = odd ? recv[w] : packed[8 * k + w];      // the even lane's row
          v2[w] = odd ? packed[8 * k + 4 + w] : recv[w];  // the odd lane's row
        }
        if (st_even)
          ptx::st_global_cs_v4(row_even + 2 * k + odd, make_uint4(v1[0], v1[1], v1[2], v1[3]));
        if (st_odd)
          ptx::st_global_cs_v4(row_odd + 2 * k + odd, make_uint4(v2[0], v2[1], v2[2], v2[3]));
      }
      if (store && p.lse != nullptr)
        p.lse[lrow] = (l > 0.f) ? (m + ptx::lg2(l)) * 0.69314718055994530942f : -INFINITY;
      // O_t has been read; the next unit's first P_t arrival (after this
      // fence) is what lets the MMA warp overwrite it.
      ptx::tc_fence_before();
    }
  }

  // ---- teardown -------------------------------------------------------------
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tessera
