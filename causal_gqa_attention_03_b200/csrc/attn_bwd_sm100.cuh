// Causal grouped-query attention backward for B200 (sm_100a): dQ, dK, dV
// from Q, K, V, O, LSE and dO.
//
// Method: the exact gradient of the forward (chain rule through the row
// softmax), computed tile by tile from the saved LSE as FlashAttention does:
//   P^T  = exp(scale*K Q^T - LSE)          (keys x queries, recomputed)
//   dP^T = V dO^T
//   dS^T = P^T * (dP^T - D),  D_i = <dO_i, O_i>
//   dV  += P^T dO,   dK += scale * dS^T Q,   dQ += scale * dS K
// The pages list the attention backward as not yet built; the forward it
// differentiates is the FlashAttention forward they name (hysenlabs.com
// Tessera review, "The kernel set and its torch fallback").
//
// Three launches:
//   1. attn_bwd_prep_kernel: D = rowsum(dO * O) in fp32; zeroes the fp32 dQ
//      accumulator.
//   2. attn_bwd_dkdv_sm100_kernel<D>: one CTA per SM walks units
//      (batch, key/value head, 128-key block), heaviest first.  A unit keeps
//      its K and V tiles in shared memory and its dK, dV accumulators in
//      tensor memory while it visits every (query head of the group, 128-row
//      query block) the keys are visible to; each visit adds its dQ partial
//      (128 rows x D, fp32) into the accumulator with vector reductions,
//      issued by a warpgroup of their own so that they overlap the next
//      visits (the reductions are bound by L2 throughput, ~4,000 cycles per
//      visit, about the time of the rest of a visit).
//   3. attn_bwd_dq_convert_kernel: dQ = bf16(scale * accumulator).
//
// Kernel 2 warp roles (384 threads):
//   warps 0-3   compute: P^T, dS^T (thread r owns key row r), then dK, dV
//   warp  4     MMA issue (lane 0) and TMEM allocation
//   warp  5     TMA producer (lane 0)
//   warps 6-7   idle
//   warps 8-11  dQ read-out: thread r loads query row r of the dQ partial from
//               TMEM, frees the columns, then adds it into the accumulator
// Tensor memory (512 columns):
//   S^T  [0, 128)      P^T (bf16 pairs) written over its first 64 columns;
//                      the dQ partial (D columns) written over it afterwards
//   dP^T [128, 256)    dS^T (bf16 pairs) written over its first 64 columns
//   dV   [256, 256 + D),  dK  [256 + D, 256 + 2 D)
// Per visit the MMA warp issues S^T = K Q^T and dP^T = V dO^T, waits for P^T
// and dS^T, then issues dV += P^T dO, dK += dS^T Q and dQp = dS K (A = dS from
// shared memory, written there by the compute warps in the 128-byte swizzled
// layout the MMA reads).  tcgen05 MMAs from one thread run in order, so dQp
// overwrites P^T only after dV has read it; the next visit's S^T waits until
// the read-out warps have loaded dQp into registers.
#pragma once

#include "attn_fwd_sm100.cuh"

namespace tessera {

enum BwdWaitCode : uint32_t {
  kErrBwdKv = 11,      // K/V tiles of a unit
  kErrBwdStage = 12,   // Q/dO stage full or empty
  kErrBwdS = 13,       // S^T and dP^T complete
  kErrBwdP = 14,       // P^T and dS^T written
  kErrBwdDq = 15,      // dQ partial complete or read out
  kErrBwdDkv = 16,     // dK, dV complete
  kErrBwdDrain = 17,
};

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
  static constexpr int DS_OFF = QDO_OFF + NST * 2 * TILE_BYTES;
  static constexpr int DS_BYTES = 128 * 128 * 2;   // dS [keys][queries], two 64-query sub-tiles
  static constexpr int LD_OFF = DS_OFF + DS_BYTES; // LSE*log2(e) [128], D [128]
  static constexpr int BAR_OFF = LD_OFF + 2 * 128 * 4;
  // kv_full, kv_empty, st_full[NST], st_empty[NST], s_full, p_full, dq_full,
  // dq_free, dkv_full, drain
  static constexpr int NBAR = 2 + 2 * NST + 6;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int ST_COL = 0;
  static constexpr int DPT_COL = 128;
  static constexpr int DV_COL = 256;
  static constexpr int DK_COL = 256 + D;
  static constexpr int THREADS = 384;
  static constexpr int MMA_WARP = 4;
  static constexpr int TMA_WARP = 5;
  static constexpr int READ_WARP0 = 8;  // warps 8-11: lane quadrant = warp % 4
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(DK_COL + D <= 512, "tensor memory budget");
};

struct BwdParams {
  int B, Hq, Hkv, T, G;
  int causal;
  float scale_log2;          // scale * log2(e)
  float scale;
  int nqb;                   // ceil(T / 128): query blocks and key blocks
  int num_units;             // B * Hkv * nqb
  const float* lse;          // [B, Hq, T]
  const float* dvec;         // D = rowsum(dO * O) [B, Hq, T]
  float* dq_acc;             // [B, Hq, T, D] fp32
  __nv_bfloat16* dk;         // [B, Hkv, T, D]
  __nv_bfloat16* dv;
  unsigned long long launch_id;
};

// Unit u: key block kb = u / (B * Hkv) (ascending: the longest causal
// extents first), batch and key/value head from the rest.
struct BwdUnit {
  int b, g, kb;
  int qb0;      // first query block that sees the keys
  int nvisit;   // G * (nqb - qb0)
};

__device__ __forceinline__ BwdUnit decode_bwd_unit(const BwdParams& p, int u) {
  BwdUnit w;
  const int bg = u % (p.B * p.Hkv);
  w.kb = u / (p.B * p.Hkv);
  w.b = bg / p.Hkv;
  w.g = bg % p.Hkv;
  w.qb0 = p.causal ? w.kb : 0;
  w.nvisit = p.G * (p.nqb - w.qb0);
  return w;
}

__device__ __forceinline__ int bwd_unit_of(const BwdParams& p, int k) {
  const int c = (k & 1) ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                        : static_cast<int>(blockIdx.x);
  const long long u = static_cast<long long>(k) * gridDim.x + c;
  return u < p.num_units ? static_cast<int>(u) : -1;
}

// Visit v of a unit: query block qb = qb0 + v / G, query head g*G + v % G.
__device__ __forceinline__ void bwd_visit(const BwdParams& p, const BwdUnit& w, int v, int& head,
                                          int& qb) {
  qb = w.qb0 + v / p.G;
  head = w.g * p.G + v % p.G;
}

// ------------------------------------------------------------------ kernel 1
// D[row] = sum_c dO[row,c] * O[row,c] (fp32), one warp per row; and the fp32
// dQ accumulator set to zero.  rows = B*Hq*T.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            float* __restrict__ dvec,
                                                            float* __restrict__ dq_acc,
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
    float4* z = reinterpret_cast<float4*>(dq_acc + r * D);
#pragma unroll
    for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ------------------------------------------------------------------ kernel 3
// dQ = bf16(scale * acc), 8 elements per thread step.
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                  __nv_bfloat16* __restrict__ dq,
                                                                  long long n8, float scale) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 r;
    r.x = ptx::pack_bf16x2(a.x * scale, a.y * scale);
    r.y = ptx::pack_bf16x2(a.z * scale, a.w * scale);
    r.z = ptx::pack_bf16x2(b.x * scale, b.y * scale);
    r.w = ptx::pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = r;
  }
}

// Byte offset of dS[key r][query c .. c + 7] (16-byte chunk) in the dS tile:
// two sub-tiles of 64 queries, each [128 keys][64 queries] with the 128-byte
// swizzle (8-row atoms of 1 KB; chunk j of row r stored at chunk j ^ (r % 8)).
__device__ __forceinline__ uint32_t ds_chunk_offset(int r, int c) {
  const int sub = c >> 6;
  const int chunk = (c & 63) >> 3;
  return static_cast<uint32_t>(sub * (128 * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                               ((chunk ^ (r & 7)) << 4));
}

// ------------------------------------------------------------------ kernel 2
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
  uint8_t* sDS = smem + C::DS_OFF;
  float* sLse = reinterpret_cast<float*>(smem + C::LD_OFF);
  float* sD = sLse + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* st_empty = st_full + C::NST;
  uint64_t* s_full = st_empty + C::NST;
  uint64_t* p_full = s_full + 1;
  uint64_t* dq_full = s_full + 2;
  uint64_t* dq_free = s_full + 3;
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
    ptx::mbar_init(p_full, 4);   // one arrival per compute warp
    ptx::mbar_init(dq_full, 1);
    ptx::mbar_init(dq_free, 4);   // one arrival per read-out warp
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
    constexpr uint32_t kIdescQ = ptx::idesc_bf16_f32(128, D, true, true);      // dQp = dS K
    constexpr uint32_t kDescHi = ptx::sdesc_sw128_hi(1024);  // SBO 1 KB, 128-B swizzle
    const uint32_t k_addr = ptx::smem_u32(sK);
    const uint32_t v_addr = ptx::smem_u32(sV);
    const uint32_t qdo_addr = ptx::smem_u32(sQdO);
    const uint32_t ds_addr = ptx::smem_u32(sDS);
    int vis = 0;    // visits issued so far (stage ring position; s_full/p_full/dq phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      if (!warp_wait(kv_full, k & 1, kErrBwdKv, p.launch_id)) break;
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        const int s = vis % C::NST;
        ok = warp_wait(&st_full[s], (vis / C::NST) & 1, kErrBwdStage, p.launch_id);
        // the previous visit's dQ partial has been read out of S^T's columns
        if (ok && vis > 0) ok = warp_wait(dq_free, (vis - 1) & 1, kErrBwdDq, p.launch_id);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t q_addr = qdo_addr + s * 2 * C::TILE_BYTES;
        const uint32_t do_addr = q_addr + C::TILE_BYTES;
        if (leader) {
          // S^T = K Q^T and dP^T = V dO^T: both operands K-major (d innermost)
          const uint32_t ka = ptx::sdesc_sw128_lo(k_addr, 16);
          const uint32_t va = ptx::sdesc_sw128_lo(v_addr, 16);
          const uint32_t qb_ = ptx::sdesc_sw128_lo(q_addr, 16);
          const uint32_t gb = ptx::sdesc_sw128_lo(do_addr, 16);
          ptx::mma_ss_lohi<0>(tmem + C::ST_COL, ka, kDescHi, qb_, kDescHi, kIdescS);
#pragma unroll
          for (int kk = 1; kk < D / 16; ++kk) {
            const uint32_t st = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
            ptx::mma_ss_lohi<1>(tmem + C::ST_COL, ka + st, kDescHi, qb_ + st, kDescHi, kIdescS);
          }
          ptx::mma_ss_lohi<0>(tmem + C::DPT_COL, va, kDescHi, gb, kDescHi, kIdescS);
#pragma unroll
          for (int kk = 1; kk < D / 16; ++kk) {
            const uint32_t st = (kk >> 2) * (C::SUB_BYTES >> 4) + (kk & 3) * 2;
            ptx::mma_ss_lohi<1>(tmem + C::DPT_COL, va + st, kDescHi, gb + st, kDescHi, kIdescS);
          }
          ptx::tc_commit(s_full);
        }
        __syncwarp();
        if (!warp_wait(p_full, vis & 1, kErrBwdP, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (leader) {
          const uint32_t first = (v == 0) ? 0u : 1u;
          // dV += P^T dO and dK += dS^T Q: A from TMEM (K = queries, 8 columns
          // per 16), B = dO / Q with queries as K and d as N (MN-major); K
          // step kk is 16 query rows = 2 KB further into the tile.
          const uint32_t gb = ptx::sdesc_sw128_lo(do_addr, C::SUB_BYTES);
          const uint32_t qb_ = ptx::sdesc_sw128_lo(q_addr, C::SUB_BYTES);
          ptx::mma_ts_lohi_rt(tmem + C::DV_COL, tmem + C::ST_COL, gb, kDescHi, kIdescG, first);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            ptx::mma_ts_lohi<1>(tmem + C::DV_COL, tmem + C::ST_COL + kk * 8, gb + kk * (2048 >> 4),
                                kDescHi, kIdescG);
          ptx::mma_ts_lohi_rt(tmem + C::DK_COL, tmem + C::DPT_COL, qb_, kDescHi, kIdescG, first);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            ptx::mma_ts_lohi<1>(tmem + C::DK_COL, tmem + C::DPT_COL + kk * 8,
                                qb_ + kk * (2048 >> 4), kDescHi, kIdescG);
          // dQp = dS K: A = dS (M = queries, K = keys) MN-major in shared
          // memory, two 64-query sub-tiles 16 KB apart; B = K (K = keys,
          // N = d) MN-major.  K step kk is 16 keys = 2 KB.
          const uint32_t da = ptx::sdesc_sw128_lo(ds_addr, C::SUB_BYTES);
          const uint32_t kb_ = ptx::sdesc_sw128_lo(k_addr, C::SUB_BYTES);
          ptx::mma_ss_lohi<0>(tmem + C::ST_COL, da, kDescHi, kb_, kDescHi, kIdescQ);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            ptx::mma_ss_lohi<1>(tmem + C::ST_COL, da + kk * (2048 >> 4), kDescHi,
                                kb_ + kk * (2048 >> 4), kDescHi, kIdescQ);
          ptx::tc_commit(dq_full);
          ptx::tc_commit(&st_empty[s]);
          if (v == w.nvisit - 1) {
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
  } else if (warp < 4) {
    // ======================= compute warps ================================
    const int row = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t st_addr = tmem + lane_base + C::ST_COL;
    const uint32_t dpt_addr = tmem + lane_base + C::DPT_COL;
    const uint32_t ds_base = ptx::smem_u32(sDS);
    const float sl2 = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    int vis = 0;
    int units = 0;
    bool ok = true;
    bool stop = false;  // every compute warp has learnt that one gave up
    for (int k = 0; !stop; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      const int key = w.kb * C::BN + row;  // this thread's key row (P^T, dS^T, dK, dV)
      const bool key_ok = key < p.T;
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        // The four compute warps meet at two named barriers per visit; a warp
        // whose wait gave up keeps taking part until the first one, where all
        // four learn of it and stop together.
        if (!ptx::bar_red_and(1, 128, ok)) {
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
          sLse[row] = (qr < p.T) ? p.lse[qrow0 + row] * kLog2e : INFINITY;
          sD[row] = (qr < p.T) ? p.dvec[qrow0 + row] : 0.f;
        }
        ptx::bar_sync_named(1, 128);
        // A warp whose wait gives up still reaches the read-out's barriers
        // below (every warp takes the same barrier sequence in each visit).
        ok = warp_wait(s_full, vis & 1, kErrBwdS, p.launch_id);
        const bool diag = p.causal && qb == w.kb;
        if (ok) {
          ptx::tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {  // 32 query columns at a time
            uint32_t sr[32], gr[32];
            ptx::tmem_ld32(st_addr + 32 * c4, sr);
            ptx::tmem_ld32(dpt_addr + 32 * c4, gr);
            ptx::tmem_ld_wait();
            ptx::reg_fence(sr);
            ptx::reg_fence(gr);
            uint32_t pp[16], dd[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float pv[2], dv[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = 32 * c4 + 2 * i + e;
                const float x = fmaf(__uint_as_float(sr[2 * i + e]), sl2, -sLse[col]);
                float pe = ptx::ex2(x);
                if (!key_ok || (diag && col < row)) pe = 0.f;  // key past T, or key > query
                pv[e] = pe;
                dv[e] = pe * (__uint_as_float(gr[2 * i + e]) - sD[col]);
              }
              pp[i] = ptx::pack_bf16x2(pv[0], pv[1]);
              dd[i] = ptx::pack_bf16x2(dv[0], dv[1]);
            }
            ptx::tmem_st16(st_addr + 16 * c4, pp);
            ptx::tmem_st16(dpt_addr + 16 * c4, dd);
            // dS row `row`, queries 32*c4 .. 32*c4+31, into the swizzled tile
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ptx::st_shared_v4(ds_base + ds_chunk_offset(row, 32 * c4 + 8 * j), dd[4 * j],
                                dd[4 * j + 1], dd[4 * j + 2], dd[4 * j + 3]);
          }
          ptx::tmem_st_wait();
          ptx::fence_proxy_async_smem();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(p_full);
        }

      }
      if (stop) break;
      // A warp whose wait gave up skips its work but walks on to the next
      // unit's first barrier, where the others learn of it.
      if (!ok) continue;

      // ---- unit epilogue: dV, scale * dK -> bf16 ------------------------------
      ok = warp_wait(dkv_full, units & 1, kErrBwdDkv, p.launch_id);
      ++units;
      if (!ok) continue;
      ptx::tc_fence_after();
      const long long krow = (static_cast<long long>(w.b) * p.Hkv + w.g) * p.T + key;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_base + (which == 0 ? C::DV_COL : C::DK_COL);
        const float mul = which == 0 ? 1.f : p.scale;
        uint4* out = reinterpret_cast<uint4*>((which == 0 ? p.dv : p.dk) + krow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
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
      // dK, dV have been read; the next unit's first P^T arrival (after this
      // fence) is what lets the MMA warp overwrite them.
      ptx::tc_fence_before();
    }
  } else if (warp >= C::READ_WARP0) {
    // ======================= dQ read-out ==================================
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // query row within the visit's block
    const uint32_t src = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::ST_COL;
    int vis = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = bwd_unit_of(p, k);
      if (u < 0) break;
      const BwdUnit w = decode_bwd_unit(p, u);
      for (int v = 0; v < w.nvisit; ++v, ++vis) {
        if (!warp_wait(dq_full, vis & 1, kErrBwdDq, p.launch_id)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t r[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(src + 32 * c, r[c]);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) ptx::reg_fence(r[c]);
        // dQp is in registers: its TMEM columns are free for the next S^T
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(dq_free);
        int head, qb;
        bwd_visit(p, w, v, head, qb);
        if (qb * C::BM + row < p.T) {
          float* dst =
              p.dq_acc + ((static_cast<long long>(w.b) * p.Hq + head) * p.T + qb * C::BM + row) * D;
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              ptx::red_add_v4_f32(dst + 32 * c + 4 * i, __uint_as_float(r[c][4 * i]),
                                  __uint_as_float(r[c][4 * i + 1]),
                                  __uint_as_float(r[c][4 * i + 2]),
                                  __uint_as_float(r[c][4 * i + 3]));
        }
      }
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
