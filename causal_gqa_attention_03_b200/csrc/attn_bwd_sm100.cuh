// Causal grouped-query attention backward for B200 (sm_100a): dQ, dK, dV
// from Q, K, V, O, LSE and dO.
//
// Method: the exact gradient of the forward (chain rule through the row
// softmax), computed tile by tile from the saved LSE as FlashAttention does:
//   P    = exp(scale*Q K^T - LSE)          (recomputed, never stored)
//   dP   = dO V^T
//   dS   = P * (dP - D),  D_i = <dO_i, O_i>
//   dV  += P^T dO,   dK += scale * dS^T Q,   dQ += scale * dS K
// The pages list the attention backward as not yet built; the forward it
// differentiates is the FlashAttention forward they name (hysenlabs.com
// Tessera review, "The kernel set and its torch fallback").
//
// Three launches (four with split key/value units, below), no atomics:
//   1. attn_bwd_prep_kernel: D = rowsum(dO * O) in fp32.
//   2. attn_bwd_dkdv_sm100_kernel<D>: one CTA per SM walks units
//      (batch, key/value head, 128-key block), heaviest first.  A unit keeps
//      its K and V tiles in shared memory and its dK, dV accumulators in
//      tensor memory while it visits every (query head of the group, 128-row
//      query block) the keys are visible to, with keys as the MMA rows:
//      S^T = K Q^T, dP^T = V dO^T, then dV += P^T dO, dK += dS^T Q.
//   3. attn_bwd_dq_sm100_kernel<D>: one CTA per SM walks units (batch, query
//      head, 128-row query block), heaviest first, like the forward: per key
//      block S = Q K^T and dP = dO V^T (both recomputed), dS, then
//      dQ += dS K into tensor memory; dQ is written once, in bf16.
// Kernel 3 recomputes two products that kernel 2 also forms (seven products
// per query/key block pair instead of five); in exchange no dQ partial ever
// goes through L2 reductions, which bound the single-kernel form (a 64 KB
// fp32 partial per visit).
//
// Few key/value units (B * Hkv * key blocks below about four per SM, e.g.
// multi-query attention) leave SMs idle and put the heaviest unit on the
// critical path.  When the caller's workspace allows, kernel 2's units are
// then cut by query heads into `split` parts whose fp32 partial dK, dV are
// summed by attn_bwd_dkv_reduce_kernel (a fourth launch) in a fixed order,
// so results stay independent of scheduling.
#pragma once

#include "attn_fwd_sm100.cuh"

namespace tessera {

enum BwdWaitCode : uint32_t {
  kErrBwdKv = 11,      // K/V tiles (kernel 2: of a unit; kernel 3: ring stages)
  kErrBwdStage = 12,   // Q/dO stages full or empty (kernel 2); Q/dO in TMEM (kernel 3)
  kErrBwdS = 13,       // S^T (kernel 2) or S (kernel 3) complete
  kErrBwdP = 14,       // P^T written (kernel 2); S or dP loaded by the compute warps (kernel 3)
  kErrBwdDq = 15,      // dS^T written, dP^T complete (kernel 2); dS written or its tile
                       // free, dP complete (kernel 3)
  kErrBwdDkv = 16,     // dK, dV (kernel 2) or dQ (kernel 3) complete
  kErrBwdDrain = 17,   // the MMAs issued, before tensor memory is freed
};

// ------------------------------------------------------------------ kernel 1
// D[row] = sum_c dO[row,c] * O[row,c] (fp32), one warp per row.  rows = B*Hq*T.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            float* __restrict__ dvec,
                                                            long long rows) {
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = wid; r < rows; r += warps) {
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(o + r * D);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(dout + r * D);
    float acc = 0.f;
#pragma unroll
    for (int c = lane; c < D / 2; c += 32) {
      const float2 a = __bfloat1622float2(o2[c]);
      const float2 b = __bfloat1622float2(g2[c]);
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dvec[r] = acc;
  }
}

// dV, dK = the sum over `split` fp32 partials [split][rows][2][D] (dV first,
// then dK, already scaled) -> bf16, in part order.  rows = B*Hkv*T.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dkv_reduce_kernel(
    const float* __restrict__ part, __nv_bfloat16* __restrict__ dk,
    __nv_bfloat16* __restrict__ dv, long long rows, int split) {
  constexpr int V4 = D / 4;  // float4 groups per row and gradient
  const long long n = rows * 2 * V4;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    const long long row = i / (2 * V4);
    const int which = static_cast<int>((i / V4) & 1);
    const int c4 = static_cast<int>(i % V4);
    const float4* src = reinterpret_cast<const float4*>(part) + i;
    float4 acc = src[0];
    for (int s = 1; s < split; ++s) {
      const float4 x = src[static_cast<long long>(s) * rows * 2 * V4];
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    __nv_bfloat16* out = (which == 0 ? dv : dk) + row * D + 4 * c4;
    uint2 packed;
    packed.x = ptx::pack_bf16x2(acc.x, acc.y);
    packed.y = ptx::pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(out) = packed;
  }
}

// ------------------------------------------------------------------ kernel 2
// Warp roles (384 threads):
//   warps 0-7   compute: warp w owns key rows 32 (w % 4) .. + 31 (TMEM lane
//               quadrant w % 4) and query columns 64 (w / 4) .. + 63 of each
//               visit: P^T, dS^T, then its D/2 columns of dK, dV.  Two warps
//               per lane quadrant overlap one's MUFU work with the other's.
//   warp  8     MMA issue (lane 0) and TMEM allocation
//   warp  9     TMA producer (lane 0)
//   warps 10-11 idle
// Tensor memory (512 columns):
//   S^T  [0, 128)      P^T (bf16 pairs) written over each half's own
//                      columns: queries 0-63 at +[0, 32), 64-127 at +[64, 96)
//   dP^T [128, 256)    dS^T (bf16 pairs) in the same split layout
//   dV   [256, 256 + D),  dK  [256 + D, 256 + 2 D)
// Per visit v the MMA warp issues, in this order:
//   (once P^T(v) is written)  dV += P^T(v) dO(v), then S^T(v+1);
//   (once dS^T(v) is written) dK += dS^T(v) Q(v), then dP^T(v+1).
// tcgen05 MMAs from one thread run in order, so S^T(v+1) overwrites P^T(v)
// only after dV has read it, and dP^T(v+1) overwrites dS^T(v) only after dK
// has; the compute warps form P^T(v+1) while dK(v) and dP^T(v+1) run.
template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BM = 128;                   // query rows per visit
  static constexpr int BN = 128;                   // keys per unit
  static constexpr int SUB = D / 64;               // 128-byte column sub-tiles per tile
  static constexpr int SUB_BYTES = 128 * 128;      // one [128 rows x 64 bf16] sub-tile
  static constexpr int TILE_BYTES = 128 * D * 2;   // one [128 x D] bf16 tile
  static constexpr int NST = (D == 128) ? 2 : 4;   // Q/dO stages
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE_BYTES;
  static constexpr int QDO_OFF = 2 * TILE_BYTES;   // stage s: Q at +2s tiles, dO at +2s+1
  static constexpr int LD_OFF = QDO_OFF + NST * 2 * TILE_BYTES;  // LSE*log2(e) [128], D [128]
  static constexpr int BAR_OFF = LD_OFF + 2 * 128 * 4;
  // kv_full, kv_empty, st_full[NST], st_empty[NST], s_full, dp_full, p_full,
  // ds_full, dkv_full, drain
  static constexpr int NBAR = 2 + 2 * NST + 6;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int ST_COL = 0;
  static constexpr int DPT_COL = 128;
  static constexpr int DV_COL = 256;
  static constexpr int DK_COL = 256 + D;
  static constexpr int THREADS = 384;
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(DK_COL + D <= 512, "tensor memory budget");
};

struct BwdParams {
  int B, Hq, Hkv, T, G;
  int causal;
  float scale_log2;          // scale * log2(e)
  float scale;
  int nqb;                   // ceil(T / 128): query blocks and key blocks
  int num_units;             // kernel 2: B * Hkv * nqb; kernel 3: B * Hq * nqb
  const float* lse;          // [B, Hq, T]
  const float* dvec;         // D = rowsum(dO * O) [B, Hq, T]
  __nv_bfloat16* dq;         // [B, Hq, T, D]
  __nv_bfloat16* dk;         // [B, Hkv, T, D]
  __nv_bfloat16* dv;
  unsigned long long launch_id;
  // kernel 2: each (batch, key/value head, key block) is cut into `split`
  // units by query heads (G / split each).  With split > 1 the units write
  // fp32 partial dV, scale * dK to dkv_part [split][B*Hkv*T][2][D], which
  // attn_bwd_dkv_reduce_kernel sums into dV, dK.
  int split;
  float* dkv_part;
  // kernel 2: 1 = batch-major unit order (set when one batch has at least
  // two units per CTA: its Q and dO then stay in L2 without costing balance)
  int kv_batch_major;
  // kernel 3: 1 = batch-major unit order (set when one batch has at least
  // two units per CTA and the whole K/V is larger than L2)
  int q_batch_major;
};

// Unit u: key block kb (ascending: the longest causal extents first), then
// batch, key/value head and query-head part; or batch first
// (kv_batch_major).
struct BwdUnit {
  int b, g, kb;
  int part;     // which G / split query heads of the group
  int qb0;      // first query block that sees the keys
  int nvisit;   // (G / split) * (nqb - qb0)
};

__device__ __forceinline__ BwdUnit decode_bwd_unit(const BwdParams& p, int u) {
  BwdUnit w;
  const int groups = p.Hkv * p.split;
  int rest;
  if (p.kv_batch_major) {
    // batch b's units (key blocks ascending, each over its heads and parts)
    // before batch b+1's, so one batch's Q and dO stay in L2
    const int per_b = groups * p.nqb;
    w.b = u / per_b;
    const int ub = u % per_b;
    rest = ub % groups;
    w.kb = ub / groups;
  } else {
    // key blocks ascending over all batches
    const int bgs = p.B * groups;
    w.kb = u / bgs;
    w.b = (u % bgs) / groups;
    rest = u % groups;
  }
  w.part = rest % p.split;
  w.g = rest / p.split;
  w.qb0 = p.causal ? w.kb : 0;
  w.nvisit = (p.G / p.split) * (p.nqb - w.qb0);
  return w;
}

// The k-th unit of this CTA (snake order over the heaviest-first list), or -1.
__device__ __forceinline__ int bwd_unit_of(const BwdParams& p, int k) {
  const int c = (k & 1) ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                        : static_cast<int>(blockIdx.x);
  const long long u = static_cast<long long>(k) * gridDim.x + c;
  return u < p.num_units ? static_cast<int>(u) : -1;
}

// Visit v of a unit: query block qb = qb0 + v / Gs, query head
// g*G + part*Gs + v % Gs, with Gs = G / split heads per part.
__device__ __forceinline__ void bwd_visit(const BwdParams& p, const BwdUnit& w, int v, int& head,
                                          int& qb) {
  const int gs = p.G / p.split;
  qb = w.qb0 + v / gs;
  head = w.g * p.G + w.part * gs + v % gs;
}

template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    attn_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  uint8_t* sQdO = smem + C::QDO_OFF;
  float* sLse = reinterpret_cast<float*>(smem + C::LD_OFF);
  float* sD = sLse + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* st_empty = st_full + C::NST;
  uint64_t* s_full = st_empty + C::NST;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* ds_full = s_full + 3;
  uint64_t* dkv_full = s_full + 4;
  uint64_t* drain = s_full + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SLOT_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(kv_full, 1);
    ptx::mbar_init(kv_empty, 1);
    for (int s = 0; s < C::NST; ++s) {
      ptx::mbar_init(&st_full[s], 1);
      ptx::mbar_init(&st_empty[s], 1);
    }
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(dp_full, 1);
    ptx::mbar_init(p_full, 8);    // one arrival per compute warp
    ptx::mbar_init(ds_full, 8);
    ptx::mbar_init(dkv_full, 1);
    ptx::mbar_init(drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == C::TMA_WARP && lane == 0) {
    ptx::prefetch_tensormap(&tm_q);
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
    ptx::prefetch_tensormap(&tm_do);
  }
  if (warp == C::MMA_WARP) {
    ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::TMA_WARP) {
    // ======================= TMA producer =================================
    const bool leader = lane == 0;
    const uint64_t keep = ptx::policy_evict_last();
    int vis = 0;  // visits loaded so far (stage ring position)
    int k = 0;
    bool ok = true;
    for (; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      // K, V of the unit once the previous unit's MMAs no longer read them
      if (!warp_wait(kv_empty, (k & 1) ^ 1u, kErrBwdKv, p.launch_id)) {
        ok = false;
        break;
      }
      const int kv_plane = w.b * p.Hkv + w.g;
      if (leader) {
        ptx::mbar_arrive_expect_tx(kv_full, 2 * C::TILE_BYTES);
        for (int c = 0; c < C::SUB; ++c) {
          ptx::tma_load_3d(sK + c * C::SUB_BYTES, &tm_k, kv_full, c * 64, w.kb * C::BN, kv_plane);
          ptx::tma_load_3d(sV + c * C::SUB_BYTES, &tm_v, kv_full, c * 64, w.kb * C::BN, kv_plane);
        }
      }
      __syncwarp();
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        const int s = vis % C::NST;
        if (!warp_wait(&st_empty[s], ((vis / C::NST) & 1) ^ 1u, kErrBwdStage, p.launch_id)) {
          ok = false;
          break;
        }
        int head, qb;
        bwd_visit(p, w, v, head, qb);
        const int plane = w.b * p.Hq + head;
        if (leader) {
          uint8_t* dst = sQdO + s * 2 * C::TILE_BYTES;
          ptx::mbar_arrive_expect_tx(&st_full[s], 2 * C::TILE_BYTES);
          for (int c = 0; c < C::SUB; ++c) {
            ptx::tma_load_3d_hint(dst + c * C::SUB_BYTES, &tm_q, &st_full[s], c * 64, qb * C::BM,
                                  plane, keep);
            ptx::tma_load_3d_hint(dst + C::TILE_BYTES + c * C::SUB_BYTES, &tm_do, &st_full[s],
                                  c * 64, qb * C::BM, plane, keep);
          }
        }
        __syncwarp();
      }
    }
    if (!ok) {
      // Gave up: let the copies already in flight land before the CTA exits.
      if (k > 0) warp_wait(kv_full, (k - 1) & 1, kErrBwdKv, p.launch_id);
      for (int i = max(0, vis - C::NST); i < vis; ++i)
        warp_wait(&st_full[i % C::NST], (i / C::NST) & 1, kErrBwdStage, p.launch_id);
    }
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issue ====================================
    const bool leader = lane == 0;
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
    constexpr uint32_t kIdescG = ptx::idesc_bf16_f32(128, D, false, true);     // dV, dK (A TMEM)
    constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);  // SBO 1 KB, 128-B swizzle
    const uint32_t k_addr = ptx::smem_u32(sK);
    const uint32_t v_addr = ptx::smem_u32(sV);
    const uint32_t qdo_addr = ptx::smem_u32(sQdO);
    // X^T = Y Z^T into TMEM column col: Y (K or V) and Z (Q or dO) both
    // K-major (d innermost); K step kk is 32 B, or the next 16 KB sub-tile.
    auto issue_t = [&](uint32_t col, uint32_t y_addr, uint32_t z_addr) {
      const uint32_t ya = ptx::sdesc_sw128_lo(y_addr, 16);
      const uint32_t zb = ptx::sdesc_sw128_lo(z_addr, 16);
      ptx::mma_ss_lohi<0>(tmem + col, ya, kDescHi, zb, kDescHi, kIdescS);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk) {
        const uint32_t st = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
        ptx::mma_ss_lohi<1>(tmem + col, ya + st, kDescHi, zb + st, kDescHi, kIdescS);
      }
    };
    // G += A^T Z into TMEM column col: A from TMEM column a_col (bf16 pairs,
    // K = queries, 8 columns per 16; queries 64-127 at +64), Z (dO or Q) with
    // queries as K and d as N (MN-major); K step kk is 16 query rows = 2 KB
    // further into the tile.
    auto issue_g = [&](uint32_t col, uint32_t a_col, uint32_t z_addr, uint32_t first) {
      const uint32_t zb = ptx::sdesc_sw128_lo(z_addr, C::SUB_BYTES);
      ptx::mma_ts_lohi_rt(tmem + col, tmem + a_col, zb, kDescHi, kIdescG, first);
#pragma unroll
      for (int kk = 1; kk < 8; ++kk)
        ptx::mma_ts_lohi<1>(tmem + col, tmem + a_col + (kk >> 2) * 64 + (kk & 3) * 8,
                            zb + kk * (2048 >> 4), kDescHi, kIdescG);
    };
    int vis = 0;    // visits issued so far (stage ring position; barrier phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      if (!warp_wait(kv_full, k & 1, kErrBwdKv, p.launch_id)) break;
      // the unit's first S^T and dP^T
      if (!warp_wait(&st_full[vis % C::NST], (vis / C::NST) & 1, kErrBwdStage, p.launch_id))
        break;
      ptx::tc_fence_after();
      if (leader) {
        const uint32_t q_addr = qdo_addr + (vis % C::NST) * 2 * C::TILE_BYTES;
        issue_t(C::ST_COL, k_addr, q_addr);
        ptx::tc_commit(s_full);
        issue_t(C::DPT_COL, v_addr, q_addr + C::TILE_BYTES);
        ptx::tc_commit(dp_full);
      }
      __syncwarp();
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        const int s = vis % C::NST;
        const int s1 = (vis + 1) % C::NST;
        const bool more = v + 1 < w.nvisit;
        const uint32_t q_addr = qdo_addr + s * 2 * C::TILE_BYTES;
        const uint32_t q1_addr = qdo_addr + s1 * 2 * C::TILE_BYTES;
        const uint32_t first = (v == 0) ? 0u : 1u;
        ok = warp_wait(p_full, vis & 1, kErrBwdP, p.launch_id);
        if (ok && more)
          ok = warp_wait(&st_full[s1], ((vis + 1) / C::NST) & 1, kErrBwdStage, p.launch_id);
        if (!ok) break;
        ptx::tc_fence_after();
        if (leader) {
          issue_g(C::DV_COL, C::ST_COL, q_addr + C::TILE_BYTES, first);  // dV += P^T dO
          if (more) {
            issue_t(C::ST_COL, k_addr, q1_addr);                         // S^T(v+1)
            ptx::tc_commit(s_full);
          }
        }
        __syncwarp();
        if (!warp_wait(ds_full, vis & 1, kErrBwdDq, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (leader) {
          issue_g(C::DK_COL, C::DPT_COL, q_addr, first);                 // dK += dS^T Q
          ptx::tc_commit(&st_empty[s]);
          if (more) {
            issue_t(C::DPT_COL, v_addr, q1_addr + C::TILE_BYTES);        // dP^T(v+1)
            ptx::tc_commit(dp_full);
          } else {
            ptx::tc_commit(dkv_full);
            ptx::tc_commit(kv_empty);
          }
        }
        __syncwarp();
      }
    }
    // Every MMA issued must finish before tensor memory is released.
    if (leader) ptx::tc_commit(drain);
    __syncwarp();
    warp_wait(drain, 0, kErrBwdDrain, p.launch_id);
  } else if (warp < 8) {
    // ======================= compute warps ================================
    // warp w: key rows 32 (w % 4) .. + 31, query columns 64 (w / 4) .. + 63
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t st_addr = tmem + lane_base + C::ST_COL + 64 * half;
    const uint32_t dpt_addr = tmem + lane_base + C::DPT_COL + 64 * half;
    const float sl2 = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    int vis = 0;
    int units = 0;
    bool ok = true;
    bool stop = false;
    for (int k = 0; !stop; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      const int key = w.kb * C::BN + row;
      const bool key_ok = key < p.T;
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        // The eight compute warps meet at two named barriers per visit; a
        // warp whose wait gave up keeps taking part until the first one,
        // where all eight learn of it and stop together.
        if (!ptx::bar_red_and(1, 256, ok)) {
          stop = true;
          break;
        }
        int head, qb;
        bwd_visit(p, w, v, head, qb);
        const long long qrow0 = (static_cast<long long>(w.b) * p.Hq + head) * p.T + qb * C::BM;
        // LSE*log2(e) and D of the visit's 128 query rows into shared memory
        // (+inf / 0 past T, so those columns of P^T and dS^T are zero).
        {
          const int qr = qb * C::BM + row;
          if (half == 0)
            sLse[row] = (qr < p.T) ? p.lse[qrow0 + row] * kLog2e : INFINITY;
          else
            sD[row] = (qr < p.T) ? p.dvec[qrow0 + row] : 0.f;
        }
        ptx::bar_sync_named(1, 256);
        const bool diag = p.causal && qb == w.kb;
        ok = warp_wait(s_full, vis & 1, kErrBwdS, p.launch_id);
        if (!ok) continue;
        ptx::tc_fence_after();
        uint32_t pr[2][32];
        ptx::tmem_ld32(st_addr, pr[0]);
        ptx::tmem_ld32(st_addr + 32, pr[1]);
        ptx::tmem_ld_wait();
        ptx::reg_fence(pr[0]);
        ptx::reg_fence(pr[1]);
        uint32_t pp[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 2 * i + e;
            const int col = 64 * half + c;
            float pe = ptx::ex2(fmaf(__uint_as_float(pr[c >> 5][c & 31]), sl2, -sLse[col]));
            if (!key_ok || (diag && col < row)) pe = 0.f;
            pv[e] = pe;
            pr[c >> 5][c & 31] = __float_as_uint(pe);
          }
          pp[i] = ptx::pack_bf16x2(pv[0], pv[1]);
        }
        ptx::tmem_st32(st_addr, pp);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full);
        ok = warp_wait(dp_full, vis & 1, kErrBwdDq, p.launch_id);
        if (!ok) continue;
        ptx::tc_fence_after();
        uint32_t gr[2][32];
        ptx::tmem_ld32(dpt_addr, gr[0]);
        ptx::tmem_ld32(dpt_addr + 32, gr[1]);
        ptx::tmem_ld_wait();
        ptx::reg_fence(gr[0]);
        ptx::reg_fence(gr[1]);
        uint32_t dd[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float dv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 2 * i + e;
            dv[e] = __uint_as_float(pr[c >> 5][c & 31]) *
                    (__uint_as_float(gr[c >> 5][c & 31]) - sD[64 * half + c]);
          }
          dd[i] = ptx::pack_bf16x2(dv[0], dv[1]);
        }
        ptx::tmem_st32(dpt_addr, dd);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ds_full);
      }
      if (stop) break;
      // A warp whose wait gave up skips its work but walks on to the next
      // unit's first barrier, where the others learn of it.
      if (!ok) continue;

      // ---- unit epilogue: dV, scale * dK -> bf16, or fp32 partials when the
      // unit is one of `split` parts (this warp's D/2 columns) ----------------
      ok = warp_wait(dkv_full, units & 1, kErrBwdDkv, p.launch_id);
      ++units;
      if (!ok) continue;
      ptx::tc_fence_after();
      constexpr int HC = D / 2;
      const long long krow = (static_cast<long long>(w.b) * p.Hkv + w.g) * p.T + key;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_base + (which == 0 ? C::DV_COL : C::DK_COL) + HC * half;
        const float mul = which == 0 ? 1.f : p.scale;
        uint4* out = reinterpret_cast<uint4*>((which == 0 ? p.dv : p.dk) + krow * D + HC * half);
        if (p.split > 1) {
          float4* part = reinterpret_cast<float4*>(
              p.dkv_part +
              ((static_cast<long long>(w.part) * p.B * p.Hkv * p.T + krow) * 2 + which) * D +
              HC * half);
#pragma unroll
          for (int c = 0; c < HC / 32; ++c) {
            uint32_t r[32];
            ptx::tmem_ld32(src + 32 * c, r);
            ptx::tmem_ld_wait();
            ptx::reg_fence(r);
            if (key_ok) {
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4)
                part[c * 8 + v4] = make_float4(
                    __uint_as_float(r[4 * v4]) * mul, __uint_as_float(r[4 * v4 + 1]) * mul,
                    __uint_as_float(r[4 * v4 + 2]) * mul, __uint_as_float(r[4 * v4 + 3]) * mul);
            }
          }
          continue;
        }
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(src + 32 * c, r);
          ptx::tmem_ld_wait();
          ptx::reg_fence(r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = ptx::pack_bf16x2(__uint_as_float(r[2 * i]) * mul,
                                     __uint_as_float(r[2 * i + 1]) * mul);
          if (key_ok) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              out[c * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                                           pk[4 * v4 + 3]);
          }
        }
      }
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

// ------------------------------------------------------------------ kernel 3
// Warp roles (384 threads):
//   warps 0-7   compute: warp w owns query rows 32 (w % 4) .. + 31 (TMEM lane
//               quadrant w % 4) and key columns 64 (w / 4) .. + 63 of each
//               S / dP tile (and d columns D/2 (w / 4) .. of Q, dO and dQ)
//   warp  8     MMA issue of S and dP (lane 0) and TMEM allocation
//   warp  9     TMA producer (lane 0): K and V tiles only
//   warp 10     MMA issue of dQ (lane 0)
//   warp 11     idle
// Tensor memory (512 columns for D = 128):
//   S    [0, 128)
//   dP   [128, 256)
//   dQ   [256, 256 + D)
//   Q    [256 + D, 256 + 3D/2)   the unit's query rows, bf16 pairs (A operand)
//   dO   [256 + 3D/2, 256 + 2D)
// Shared memory: the K/V ring and one dS tile [128 rows][128 keys] bf16 in
// the 128-byte-swizzled K-major layout (two 64-key sub-tiles), the A operand
// of dQ += dS K.
// Q and dO are the A operands of S = Q K^T and dP = dO V^T straight from
// tensor memory, so those products read only K or V from shared memory.  No
// product's input aliases another's output, so each is issued as soon as its
// inputs are free: per key block j
//   warp 8 issues S(j+1)  once the compute warps have loaded S(j),
//          and dP(j+1)    once they have loaded dP(j);
//   warp 10 issues dQ += dS(j) K_j  once dS(j) is in shared memory.
// The two issuers need no ordering between them: S and dP write only their
// own columns and read Q, dO, K, V; dQ reads dS and K and writes only dQ.
// K_j, read by S(j) and dQ(j), is released by warp 10 after dQ(j): S(j) is
// complete by then (the compute warps loaded its result before writing dS).
// A single issuer spent most of each block waiting on barriers in a fixed
// order; two let dQ(j) go out while warp 8 waits for the next S / dP slot.
template <int D>
struct DqCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int BM = 128;                  // query rows per unit
  static constexpr int BN = 128;                  // keys per block
  static constexpr int SUB = D / 64;
  static constexpr int SUB_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NSTAGE = (D == 128) ? 6 : 12;  // K/V ring (K_j, V_j alternate)
  static constexpr int KV_OFF = 0;
  static constexpr int DS_OFF = KV_OFF + NSTAGE * TILE_BYTES;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int BAR_OFF = DS_OFF + DS_BYTES;
  // kv_full[NSTAGE], kv_empty[NSTAGE], q_ready, s_full, s_free, dp_full,
  // dp_free, ds_full, ds_free, dq_full, drain (warp 8), drain (warp 10)
  static constexpr int NBAR = 2 * NSTAGE + 10;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = 128;
  static constexpr int DQ_COL = 256;
  static constexpr int Q_COL = 256 + D;
  static constexpr int DO_COL = 256 + D + D / 2;
  static constexpr int THREADS = 384;
  static constexpr int MMA_WARP = 8;
  static constexpr int TMA_WARP = 9;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(DO_COL + D / 2 <= 512, "tensor memory budget");
};

// Unit u of kernel 3: step = u / (B * Hq) from the heaviest query block down
// (causal); batch and query head from the rest.
struct DqUnit {
  int b, h, qb, n;  // n: key blocks visited
};

__device__ __forceinline__ DqUnit decode_dq_unit(const BwdParams& p, int u) {
  DqUnit w;
  int step;
  if (p.q_batch_major) {
    // batch b's units (heaviest first) before batch b+1's: one batch's K and
    // V stay in L2
    const int per_b = p.Hq * p.nqb;
    w.b = u / per_b;
    const int ub = u % per_b;
    step = ub / p.Hq;
    w.h = ub % p.Hq;
  } else {
    const int bh = u % (p.B * p.Hq);
    step = u / (p.B * p.Hq);
    w.b = bh / p.Hq;
    w.h = bh % p.Hq;
  }
  w.qb = p.nqb - 1 - step;
  w.n = p.causal ? w.qb + 1 : p.nqb;
  return w;
}

// Byte offset of row r, columns c .. c + 7 (one 16-byte chunk) in a
// [128 rows][128 columns] bf16 tile stored as two 64-column sub-tiles with the
// 128-byte swizzle (8-row atoms of 1 KB; chunk j of row r at chunk j ^ (r % 8)).
__device__ __forceinline__ uint32_t ds_chunk_offset(int r, int c) {
  const int sub = c >> 6;
  const int chunk = (c & 63) >> 3;
  return static_cast<uint32_t>(sub * (128 * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                               ((chunk ^ (r & 7)) << 4));
}

// P of one row (this thread) over 64 key columns of a block: s holds the raw
// scores on entry and P (fp32) on return.  Masked keys (kv0 + c > lim) get
// P = 0 when kMasked.
template <bool kMasked>
__device__ __forceinline__ void dq_p_tile(uint32_t (&s)[2][32], float sl2, float lse_l2,
                                          int kv0, int lim) {
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    float pe = ptx::ex2(fmaf(__uint_as_float(s[c >> 5][c & 31]), sl2, -lse_l2));
    if (kMasked && kv0 + c > lim) pe = 0.f;
    s[c >> 5][c & 31] = __float_as_uint(pe);
  }
}

// D/2 bf16 of one row (16-byte aligned) as D/4 packed pairs, or zeros.
template <int D>
__device__ __forceinline__ void load_row_half(const __nv_bfloat16* src, bool ok,
                                              uint32_t (&r)[D / 4]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < D / 16; ++i) {
    const uint4 v = ok ? __ldg(s4 + i) : make_uint4(0u, 0u, 0u, 0u);
    r[4 * i] = v.x;
    r[4 * i + 1] = v.y;
    r[4 * i + 2] = v.z;
    r[4 * i + 3] = v.w;
  }
}

template <int D>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
    attn_bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v,
                             const __nv_bfloat16* __restrict__ q,
                             const __nv_bfloat16* __restrict__ dout, const BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t* sKV = smem + C::KV_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + C::NSTAGE;
  uint64_t* q_ready = kv_empty + C::NSTAGE;
  uint64_t* s_full = q_ready + 1;
  uint64_t* s_free = q_ready + 2;
  uint64_t* dp_full = q_ready + 3;
  uint64_t* dp_free = q_ready + 4;
  uint64_t* ds_full = q_ready + 5;
  uint64_t* ds_free = q_ready + 6;
  uint64_t* dq_full = q_ready + 7;
  uint64_t* drain = q_ready + 8;
  uint64_t* drain2 = q_ready + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SLOT_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTAGE; ++s) {
      ptx::mbar_init(&kv_full[s], 1);
      ptx::mbar_init(&kv_empty[s], 1);
    }
    ptx::mbar_init(q_ready, 8);   // one arrival per compute warp
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(s_free, 8);
    ptx::mbar_init(dp_full, 1);
    ptx::mbar_init(dp_free, 8);
    ptx::mbar_init(ds_full, 8);
    ptx::mbar_init(ds_free, 1);
    ptx::mbar_init(dq_full, 1);
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(drain2, 1);
    ptx::fence_mbar_init();
  }
  if (warp == C::TMA_WARP && lane == 0) {
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

  if (warp == C::TMA_WARP) {
    // ======================= TMA producer =================================
    // Per unit: K_0, V_0, K_1, V_1, ... into the ring.
    const bool leader = lane == 0;
    const uint64_t keep = ptx::policy_evict_last();
    int idx = 0;  // K/V tiles loaded so far (ring position)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const DqUnit w = decode_dq_unit(p, u);
      const int kv_plane = w.b * p.Hkv + w.h / p.G;
      for (int i = 0; i < 2 * w.n; ++i, ++idx) {
        const int s = idx % C::NSTAGE;
        if (!warp_wait(&kv_empty[s], ((idx / C::NSTAGE) & 1) ^ 1u, kErrBwdKv, p.launch_id)) {
          ok = false;
          break;
        }
        if (leader) {
          ptx::mbar_arrive_expect_tx(&kv_full[s], C::TILE_BYTES);
          const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
          for (int c = 0; c < C::SUB; ++c)
            ptx::tma_load_3d_hint(sKV + s * C::TILE_BYTES + c * C::SUB_BYTES, map, &kv_full[s],
                                  c * 64, (i >> 1) * C::BN, kv_plane, keep);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      // Gave up: let the copies already in flight land before the CTA exits.
      for (int i = max(0, idx - C::NSTAGE); i < idx; ++i)
        warp_wait(&kv_full[i % C::NSTAGE], (i / C::NSTAGE) & 1, kErrBwdKv, p.launch_id);
    }
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issue: S and dP ==========================
    const bool leader = lane == 0;
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, false, false);  // S, dP
    constexpr uint32_t kIdescQ = ptx::idesc_bf16_f32(128, D, false, true);     // dQ
    constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);
    const uint32_t kv_addr = ptx::smem_u32(sKV);
    const uint32_t ds_addr = ptx::smem_u32(smem + C::DS_OFF);
    // X = A Z^T into TMEM column col: A from TMEM column a_col (bf16 pairs, K =
    // d, 8 columns per 16), Z (K or V) K-major in shared memory; K step kk is
    // 32 B, or the next 16 KB sub-tile.
    auto issue_x = [&](uint32_t col, uint32_t a_col, uint32_t z_addr) {
      const uint32_t zb = ptx::sdesc_sw128_lo(z_addr, 16);
      ptx::mma_ts_lohi<0>(tmem + col, tmem + a_col, zb, kDescHi, kIdescS);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk) {
        const uint32_t st = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
        ptx::mma_ts_lohi<1>(tmem + col, tmem + a_col + kk * 8, zb + st, kDescHi, kIdescS);
      }
    };
    auto stage = [&](int i) { return kv_addr + (i % C::NSTAGE) * C::TILE_BYTES; };
    auto kv_ready = [&](int i) {
      return warp_wait(&kv_full[i % C::NSTAGE], (i / C::NSTAGE) & 1, kErrBwdKv, p.launch_id);
    };
    int base = 0;  // ring position of the unit's K_0
    int sc = 0;    // key blocks so far (barrier phases)
    int units = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const DqUnit w = decode_dq_unit(p, u);
      // Q and dO of the unit are in tensor memory; S(0), dP(0)
      ok = warp_wait(q_ready, units & 1, kErrBwdStage, p.launch_id) && kv_ready(base) &&
           kv_ready(base + 1);
      ++units;
      if (!ok) break;
      ptx::tc_fence_after();
      if (leader) {
        issue_x(C::S_COL, C::Q_COL, stage(base));
        ptx::tc_commit(s_full);
        issue_x(C::DP_COL, C::DO_COL, stage(base + 1));
        ptx::tc_commit(dp_full);
        ptx::tc_commit(&kv_empty[(base + 1) % C::NSTAGE]);  // V_0: dP(0) was its reader
      }
      __syncwarp();
      for (int j = 0; j < w.n; ++j, ++sc) {
        const int kidx = base + 2 * j;
        const bool more = j + 1 < w.n;
        // S(j+1) once every compute warp has loaded S(j)
        ok = warp_wait(s_free, sc & 1, kErrBwdP, p.launch_id);
        if (ok && more) ok = kv_ready(kidx + 2);
        if (!ok) break;
        ptx::tc_fence_after();
        if (leader && more) {
          issue_x(C::S_COL, C::Q_COL, stage(kidx + 2));
          ptx::tc_commit(s_full);
        }
        __syncwarp();
        // dP(j+1) once every compute warp has loaded dP(j)
        ok = warp_wait(dp_free, sc & 1, kErrBwdP, p.launch_id);
        if (ok && more) ok = kv_ready(kidx + 3);
        if (!ok) break;
        ptx::tc_fence_after();
        if (leader && more) {
          issue_x(C::DP_COL, C::DO_COL, stage(kidx + 3));
          ptx::tc_commit(dp_full);
          ptx::tc_commit(&kv_empty[(kidx + 3) % C::NSTAGE]);  // V_{j+1}: dP(j+1) its reader
        }
        __syncwarp();
      }
      base += 2 * w.n;
    }
    if (leader) ptx::tc_commit(drain);
    __syncwarp();
    warp_wait(drain, 0, kErrBwdDrain, p.launch_id);
  } else if (warp == 10) {
    // ======================= dQ MMA issue =================================
    const bool leader = lane == 0;
    constexpr uint32_t kIdescQ = ptx::idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);
    const uint32_t kv_addr = ptx::smem_u32(sKV);
    const uint32_t ds_addr = ptx::smem_u32(smem + C::DS_OFF);
    int base = 0, sc = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const DqUnit w = decode_dq_unit(p, u);
      for (int j = 0; j < w.n; ++j, ++sc) {
        const int kidx = base + 2 * j;
        ok = warp_wait(ds_full, sc & 1, kErrBwdDq, p.launch_id);
        if (!ok) break;
        ptx::tc_fence_after();
        if (leader) {
          const uint32_t da = ptx::sdesc_sw128_lo(ds_addr, 16);
          const uint32_t kb = ptx::sdesc_sw128_lo(kv_addr + (kidx % C::NSTAGE) * C::TILE_BYTES, C::SUB_BYTES);
          ptx::mma_ss_lohi_rt(tmem + C::DQ_COL, da, kDescHi, kb, kDescHi, kIdescQ, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            ptx::mma_ss_lohi<1>(tmem + C::DQ_COL, da + (kk >> 2) * (16384 >> 4) + (kk & 3) * 2,
                                kDescHi, kb + kk * (2048 >> 4), kDescHi, kIdescQ);
          ptx::tc_commit(ds_free);
          ptx::tc_commit(&kv_empty[kidx % C::NSTAGE]);
          if (j == w.n - 1) ptx::tc_commit(dq_full);
        }
        __syncwarp();
      }
      base += 2 * w.n;
    }
    if (leader) ptx::tc_commit(drain2);
    __syncwarp();
    warp_wait(drain2, 0, kErrBwdDrain, p.launch_id);
  } else if (warp < 8) {
    // ======================= compute warps ================================
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int r = quad * 32 + lane;  // query row within the block
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int HC = D / 2;  // d columns of Q, dO, dQ per warp
    const uint32_t ds_base = ptx::smem_u32(smem + C::DS_OFF);
    int sc = 0;
    int units = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const DqUnit w = decode_dq_unit(p, u);
      const int q_row = w.qb * C::BM + r;
      const bool row_ok = q_row < p.T;
      const long long grow = (static_cast<long long>(w.b) * p.Hq + w.h) * p.T + q_row;
      const float lse_l2 = row_ok ? p.lse[grow] * kLog2e : INFINITY;
      const float dval = row_ok ? p.dvec[grow] : 0.f;
      const int lim = p.causal ? min(q_row, p.T - 1) : p.T - 1;  // last visible key
      // This row's halves of Q and dO into tensor memory (zeros past T).  The
      // previous unit's S and dP have completed: their results were loaded.
      {
        uint32_t qa[D / 4], ga[D / 4];
        load_row_half<D>(q + grow * D + HC * half, row_ok, qa);
        load_row_half<D>(dout + grow * D + HC * half, row_ok, ga);
        if constexpr (D == 128) {
          ptx::tmem_st32(tmem + lane_base + C::Q_COL + 32 * half, qa);
          ptx::tmem_st32(tmem + lane_base + C::DO_COL + 32 * half, ga);
        } else {
          ptx::tmem_st16(tmem + lane_base + C::Q_COL + 16 * half, qa);
          ptx::tmem_st16(tmem + lane_base + C::DO_COL + 16 * half, ga);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(q_ready);
      }
      for (int j = 0; j < w.n; ++j, ++sc) {
        if (!warp_wait(s_full, sc & 1, kErrBwdS, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t sv[2][32];
        ptx::tmem_ld32(tmem + lane_base + C::S_COL + 64 * half, sv[0]);
        ptx::tmem_ld32(tmem + lane_base + C::S_COL + 64 * half + 32, sv[1]);
        ptx::tmem_ld_wait();
        ptx::reg_fence(sv[0]);
        ptx::reg_fence(sv[1]);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(s_free);
        const int kv0 = j * C::BN + 64 * half;
        const int row0 = w.qb * C::BM + quad * 32;  // this warp's first query row
        const bool edge = p.causal ? (kv0 + 63 > row0) : (kv0 + 64 > p.T);
        if (edge)
          dq_p_tile<true>(sv, sl2, lse_l2, kv0, lim);
        else
          dq_p_tile<false>(sv, sl2, lse_l2, kv0, lim);
        if (!warp_wait(dp_full, sc & 1, kErrBwdDq, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t gv[2][32];
        const uint32_t dp_addr = tmem + lane_base + C::DP_COL + 64 * half;
        ptx::tmem_ld32(dp_addr, gv[0]);
        ptx::tmem_ld32(dp_addr + 32, gv[1]);
        ptx::tmem_ld_wait();
        ptx::reg_fence(gv[0]);
        ptx::reg_fence(gv[1]);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(dp_free);
        uint32_t ds[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c0 = 2 * i, c1 = 2 * i + 1;
          ds[i] = ptx::pack_bf16x2(
              __uint_as_float(sv[c0 >> 5][c0 & 31]) * (__uint_as_float(gv[c0 >> 5][c0 & 31]) - dval),
              __uint_as_float(sv[c1 >> 5][c1 & 31]) * (__uint_as_float(gv[c1 >> 5][c1 & 31]) - dval));
        }
        // dS row r, keys 64 half .. + 63, into the swizzled tile once dQ(j-1)
        // has read the previous one
        if (!warp_wait(ds_free, (sc & 1) ^ 1u, kErrBwdDq, p.launch_id)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_shared_v4(ds_base + ds_chunk_offset(r, 64 * half + 8 * c), ds[4 * c],
                            ds[4 * c + 1], ds[4 * c + 2], ds[4 * c + 3]);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ds_full);
      }
      if (!ok) break;

      // ---- epilogue: dQ = scale * acc -> bf16 -------------------------------
      if (!warp_wait(dq_full, units & 1, kErrBwdDkv, p.launch_id)) break;
      ++units;
      ptx::tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(p.dq + grow * D + HC * half);
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        uint32_t a[32];
        ptx::tmem_ld32(tmem + lane_base + C::DQ_COL + HC * half + 32 * c, a);
        ptx::tmem_ld_wait();
        ptx::reg_fence(a);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = ptx::pack_bf16x2(__uint_as_float(a[2 * i]) * p.scale,
                                   __uint_as_float(a[2 * i + 1]) * p.scale);
        if (row_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[c * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                                         pk[4 * v4 + 3]);
        }
      }
      // dQ has been read; the next unit's first dS arrival (after this fence)
      // is what lets the MMA warp overwrite it.
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
