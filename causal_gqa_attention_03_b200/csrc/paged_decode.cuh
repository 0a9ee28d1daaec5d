// One decoding step of grouped-query attention over a block-paged key/value
// cache (the serving engine's paged KV cache of the Tessera pages), for B200
// (sm_100a).
//
// Sequence b has seq_lens[b] cached tokens; token j lives in physical block
// block_table[b][j / bs], row j % bs.  Query head h (one query row per
// sequence) attends to all of them through key/value head h / G:
//   O[b,h,:] = sum_j softmax_j(scale * <q[b,h], k_j>) v_j,  LSE = log-sum-exp.
//
// The step reads every cached key and value once and does a few flops per
// byte, so it is bound by HBM bandwidth and runs on the FP32 pipes.  Split-KV
// (one CTA per 128-token chunk of one sequence and key/value head, for GT of
// its G query heads) and a merge:
//   1. paged_decode_partial_kernel: the pages of the chunk come into shared
//      memory by TMA (boxes of 64 columns x R rows, R = min(bs, 128), with the
//      128-byte swizzle, evict-first in L2).  Scores: a thread per token and
//      column half, reading its swizzled K row without bank conflicts while
//      q is a shared-memory broadcast.  Per head: the chunk max m and
//      p = 2^(s - m), l = sum p.  Values: threads over 4-column groups and
//      token slices, then a sum over the slices.  Writes the unnormalised
//      partial o, m and l per (b, h, chunk).
//   2. paged_decode_merge_kernel: a warp per (b, h) combines the chunks:
//      M = max m_c, L = sum l_c 2^(m_c - M), O = sum o_c 2^(m_c - M) / L.
// Scores are in log2 units (q is pre-multiplied by scale * log2(e)).
// A sequence length above the step's maximum, or a block id outside the
// cache among the pages a chunk needs, sets a device error code; such a
// sequence (chunk) contributes nothing and nothing outside the cache is read.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd_sm100.cuh"

namespace tessera {

constexpr uint32_t kErrDecodeInput = 20;  // a sequence length or block id out of range
constexpr uint32_t kErrDecodeWait = 21;   // the wait for a chunk's pages gave up

constexpr int kDecodeChunk = 128;    // tokens per CTA
constexpr int kDecodeThreads = 256;  // 8 warps

template <int D, int GT>
struct DecodeCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static_assert(GT == 1 || GT == 2 || GT == 4 || GT == 8, "1, 2, 4 or 8 heads per CTA");
  static constexpr int CH = kDecodeChunk;
  static constexpr int NH = D / 64;      // 64-column halves (one TMA box width each)
  static constexpr int HALF = CH * 128;  // bytes of one half-tile [CH rows][64 cols]
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NH * HALF;
  static constexpr int Q_OFF = 2 * NH * HALF;             // float [GT][D]
  static constexpr int SP_OFF = Q_OFF + GT * D * 4;       // float [2][GT][CH] partial scores
  static constexpr int P_OFF = SP_OFF + 2 * GT * CH * 4;  // float [CH][GT]
  static constexpr int ML_OFF = P_OFF + CH * GT * 4;      // float m[GT], l[GT]
  static constexpr int BAR_OFF = ML_OFF + 64;             // 2 mbarriers + a flag
  static constexpr int BYTES = BAR_OFF + 32;
  static constexpr int SMEM = BYTES + 1024;               // slack for the 1024-byte alignment
  // the sums over token slices reuse the K tile: [8 warps][GT][D] floats
  static_assert(8 * GT * D * 4 <= NH * HALF, "slice sums fit in the K tile");
  static_assert(GT * D / 4 <= kDecodeThreads, "one output group per thread");
};

struct DecodeParams {
  const __nv_bfloat16* q;      // [B, Hq, D]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  __nv_bfloat16* o;            // [B, Hq, D]
  float* lse;                  // [B, Hq] or null
  float* part_o;               // [B*Hq, nch, D]  unnormalised partial outputs
  float* part_ml;              // [B*Hq, nch, 2]  chunk max (log2 units) and sum
  int B, Hq, Hkv, G, bs, rows_per_box, max_blocks, num_blocks, max_seq_len, nch, zgroups;
  float scale_log2;  // scale * log2(e)
  unsigned long long launch_id;
};

__device__ __forceinline__ void decode_error(const DecodeParams& p, uint32_t code) {
  atomicCAS(&g_tessera_err, 0ull, ((p.launch_id & 0xffffffffull) << 32) | code);
}

// Valid length of sequence b (0, with the error recorded, when out of range).
__device__ __forceinline__ int decode_len(const DecodeParams& p, int b) {
  const int n = p.seq_lens[b];
  if (n < 0 || n > p.max_seq_len) {
    decode_error(p, kErrDecodeInput);
    return 0;
  }
  return n;
}

// Bounded wait on an mbarrier phase (no other CTA's state matters here).
__device__ __forceinline__ bool decode_wait(uint64_t* bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && ptx::globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float (&f)[8]) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16);
  f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16);
  f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Byte offset, in a [rows][64 cols] bf16 half-tile written by TMA with the
// 128-byte swizzle (1024-byte aligned), of the 16-byte chunk c of row r.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <int GT>
__device__ __forceinline__ void decode_empty_partial(const DecodeParams& p, long long head0,
                                                     int c) {
  if (threadIdx.x < GT) {
    float* ml = p.part_ml + ((head0 + threadIdx.x) * p.nch + c) * 2;
    ml[0] = -INFINITY;
    ml[1] = 0.f;
  }
}

template <int D, int GT>
__global__ void __launch_bounds__(kDecodeThreads)
    paged_decode_partial_kernel(const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeCfg<D, GT>;
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  float* sq = reinterpret_cast<float*>(sm + C::Q_OFF);
  float* sp = reinterpret_cast<float*>(sm + C::SP_OFF);
  float* spp = reinterpret_cast<float*>(sm + C::P_OFF);
  float* sml = reinterpret_cast<float*>(sm + C::ML_OFF);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  int* sflag = reinterpret_cast<int*>(sm + C::BAR_OFF + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.nch));
  const int rest = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.nch));
  const int z = rest % p.zgroups;
  const int bg = rest / p.zgroups;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int n = decode_len(p, b);
  const int t0 = c * C::CH;
  if (t0 >= n) return;  // past the sequence's last chunk: the merge reads nothing here
  const int nt = min(C::CH, n - t0);
  const int R = p.rows_per_box;
  const int npg = (nt + R - 1) / R;  // boxes (pages or parts of one) the chunk needs, <= CH / 8
  const long long head0 = static_cast<long long>(b) * p.Hq + g * p.G + z * GT;

  // warp 0 reads the chunk's block ids and sets up the barriers
  int blk = 0;
  if (warp == 0) {
    bool bad = false;
    if (lane < npg) {
      const int tok = t0 + lane * R;
      blk = p.block_table[static_cast<long long>(b) * p.max_blocks + tok / p.bs];
      bad = blk < 0 || blk >= p.num_blocks;
    }
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      *sflag = any_bad ? 1 : 0;
      if (any_bad) decode_error(p, kErrDecodeInput);
      ptx::mbar_init(&bar[0], 1);
      ptx::mbar_init(&bar[1], 1);
      ptx::fence_mbar_init();
    }
  }
  __syncthreads();
  if (*sflag) {  // a page of this chunk is not in the cache: the chunk contributes nothing
    decode_empty_partial<GT>(p, head0, c);
    return;
  }
  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(npg * R * D * 2);
      ptx::mbar_arrive_expect_tx(&bar[0], bytes);
      ptx::mbar_arrive_expect_tx(&bar[1], bytes);
    }
    __syncwarp();
    if (lane < npg) {
      const uint64_t pol = ptx::policy_evict_first();
      const int tok = t0 + lane * R;
      const int row = (blk * p.Hkv + g) * p.bs + tok % p.bs;
#pragma unroll
      for (int h = 0; h < C::NH; ++h)
        ptx::tma_load_2d_hint(sm + C::K_OFF + h * C::HALF + lane * R * 128, &tm_k, &bar[0],
                              64 * h, row, pol);
#pragma unroll
      for (int h = 0; h < C::NH; ++h)
        ptx::tma_load_2d_hint(sm + C::V_OFF + h * C::HALF + lane * R * 128, &tm_v, &bar[1],
                              64 * h, row, pol);
    }
  }
  // q of the CTA's heads, in log2 units
  for (int i = tid; i < GT * D; i += kDecodeThreads)
    sq[i] = __bfloat162float(p.q[head0 * D + i]) * p.scale_log2;
  __syncthreads();

  bool ok = decode_wait(&bar[0], 0);
  ok = __syncthreads_and(ok) != 0;
  if (!ok) {
    // record, let the copies in flight land (bounded), leave the partial empty
    if (tid == 0) {
      decode_error(p, kErrDecodeWait);
      decode_wait(&bar[0], 0);
      decode_wait(&bar[1], 0);
    }
    decode_empty_partial<GT>(p, head0, c);
    return;
  }

  // 1. partial scores: thread = (column half, token)
  {
    const int part = warp >> 2;
    const int t = ((warp & 3) << 5) | lane;
    float s[GT];
#pragma unroll
    for (int gh = 0; gh < GT; ++gh) s[gh] = t < nt ? 0.f : -INFINITY;
    if (t < nt) {
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const int gc = part * (D / 16) + j;  // 16-byte chunk of the row (8 columns)
        const uint4 u = *reinterpret_cast<const uint4*>(sm + C::K_OFF + (gc >> 3) * C::HALF +
                                                        sw128(t, gc & 7));
        float kf[8];
        bf16x8_to_f32(u, kf);
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) {
          const float4 qa = *reinterpret_cast<const float4*>(sq + gh * D + gc * 8);
          const float4 qb = *reinterpret_cast<const float4*>(sq + gh * D + gc * 8 + 4);
          s[gh] = fmaf(kf[0], qa.x, s[gh]);
          s[gh] = fmaf(kf[1], qa.y, s[gh]);
          s[gh] = fmaf(kf[2], qa.z, s[gh]);
          s[gh] = fmaf(kf[3], qa.w, s[gh]);
          s[gh] = fmaf(kf[4], qb.x, s[gh]);
          s[gh] = fmaf(kf[5], qb.y, s[gh]);
          s[gh] = fmaf(kf[6], qb.z, s[gh]);
          s[gh] = fmaf(kf[7], qb.w, s[gh]);
        }
      }
    }
#pragma unroll
    for (int gh = 0; gh < GT; ++gh) sp[(part * GT + gh) * C::CH + t] = s[gh];
  }
  // V must have landed before step 3; waiting here overlaps it with step 2
  ok = decode_wait(&bar[1], 0);
  ok = __syncthreads_and(ok) != 0;
  if (!ok) {
    if (tid == 0) decode_error(p, kErrDecodeWait);
    decode_empty_partial<GT>(p, head0, c);
    return;
  }

  // 2. per head (warp gh): chunk max m, p = 2^(s - m), l = sum p
  if (warp < GT) {
    const int gh = warp;
    float sv[C::CH / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < C::CH / 32; ++j) {
      const int t = lane + 32 * j;
      sv[j] = sp[gh * C::CH + t] + sp[(GT + gh) * C::CH + t];
      mx = fmaxf(mx, sv[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < C::CH / 32; ++j) {
      const float e = ptx::ex2(sv[j] - mx);  // masked tokens: 2^-inf = 0
      spp[(lane + 32 * j) * GT + gh] = e;
      sum += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
      sml[gh] = mx;
      sml[GT + gh] = sum;
    }
  }
  __syncthreads();

  // 3. o[gh][4cg .. 4cg+3] = sum_i p[i][gh] v_i: lanes over 4-column groups,
  // token slices over warps (and lane halves when D = 64)
  {
    constexpr int LPR = D / 4;       // lanes per V row
    constexpr int RPW = 32 / LPR;    // rows per warp step
    constexpr int STRIDE = 8 * RPW;  // token stride of a slice
    const int cg = lane % LPR;
    const int r = lane / LPR;
    const int gc = cg >> 1;
    const uint32_t vcol =
        static_cast<uint32_t>(C::V_OFF + (gc >> 3) * C::HALF + ((cg & 1) << 3));
    float acc[GT][4];
#pragma unroll
    for (int gh = 0; gh < GT; ++gh) acc[gh][0] = acc[gh][1] = acc[gh][2] = acc[gh][3] = 0.f;
#pragma unroll 4
    for (int i = warp * RPW + r; i < nt; i += STRIDE) {
      const uint2 u = *reinterpret_cast<const uint2*>(sm + vcol + sw128(i, gc & 7));
      const float v0 = __uint_as_float(u.x << 16), v1 = __uint_as_float(u.x & 0xffff0000u);
      const float v2 = __uint_as_float(u.y << 16), v3 = __uint_as_float(u.y & 0xffff0000u);
      float pw[GT];
      if constexpr (GT >= 4) {
#pragma unroll
        for (int q4 = 0; q4 < GT / 4; ++q4) {
          const float4 x = *reinterpret_cast<const float4*>(spp + i * GT + 4 * q4);
          pw[4 * q4] = x.x;
          pw[4 * q4 + 1] = x.y;
          pw[4 * q4 + 2] = x.z;
          pw[4 * q4 + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int gh = 0; gh < GT; ++gh) pw[gh] = spp[i * GT + gh];
      }
#pragma unroll
      for (int gh = 0; gh < GT; ++gh) {
        acc[gh][0] = fmaf(pw[gh], v0, acc[gh][0]);
        acc[gh][1] = fmaf(pw[gh], v1, acc[gh][1]);
        acc[gh][2] = fmaf(pw[gh], v2, acc[gh][2]);
        acc[gh][3] = fmaf(pw[gh], v3, acc[gh][3]);
      }
    }
    if constexpr (RPW == 2) {
#pragma unroll
      for (int gh = 0; gh < GT; ++gh)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[gh][e] += __shfl_xor_sync(0xffffffffu, acc[gh][e], 16);
    }
    float* red = reinterpret_cast<float*>(sm + C::K_OFF);  // K is no longer read
    if (r == 0) {
#pragma unroll
      for (int gh = 0; gh < GT; ++gh)
        *reinterpret_cast<float4*>(red + (warp * GT + gh) * D + 4 * cg) =
            make_float4(acc[gh][0], acc[gh][1], acc[gh][2], acc[gh][3]);
    }
    __syncthreads();
    if (tid < GT * D / 4) {
      const int gh = tid / (D / 4), col = 4 * (tid % (D / 4));
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 x = *reinterpret_cast<const float4*>(red + (w * GT + gh) * D + col);
        a.x += x.x;
        a.y += x.y;
        a.z += x.z;
        a.w += x.w;
      }
      *reinterpret_cast<float4*>(p.part_o + ((head0 + gh) * p.nch + c) * D + col) = a;
    }
    if (tid < GT) {
      float* ml = p.part_ml + ((head0 + tid) * p.nch + c) * 2;
      ml[0] = sml[tid];
      ml[1] = sml[GT + tid];
    }
  }
}

// A warp per (b, h): combine the sequence's chunks.  Lanes own D/32 columns.
template <int D>
__global__ void __launch_bounds__(256) paged_decode_merge_kernel(const DecodeParams p) {
  constexpr int PER = D / 32;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(p.B) * p.Hq) return;
  const int b = static_cast<int>(wid / p.Hq);
  const int n = decode_len(p, b);
  const int nc = (n + kDecodeChunk - 1) / kDecodeChunk;
  const float* ml = p.part_ml + wid * p.nch * 2;
  float M = -INFINITY;
  for (int c = lane; c < nc; c += 32) M = fmaxf(M, ml[2 * c]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const float* po = p.part_o + wid * p.nch * D + lane * PER;
  for (int c = 0; c < nc; ++c) {
    const float m = ml[2 * c];
    if (m == -INFINITY) continue;  // an empty chunk (its pages were not in the cache)
    const float w = ptx::ex2(m - M);
    L = fmaf(w, ml[2 * c + 1], L);
    if constexpr (PER == 4) {
      const float4 x = *reinterpret_cast<const float4*>(po + static_cast<long long>(c) * D);
      acc[0] = fmaf(w, x.x, acc[0]);
      acc[1] = fmaf(w, x.y, acc[1]);
      acc[2] = fmaf(w, x.z, acc[2]);
      acc[3] = fmaf(w, x.w, acc[3]);
    } else {
      const float2 x = *reinterpret_cast<const float2*>(po + static_cast<long long>(c) * D);
      acc[0] = fmaf(w, x.x, acc[0]);
      acc[1] = fmaf(w, x.y, acc[1]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* dst = p.o + wid * D + lane * PER;
  if constexpr (PER == 4) {
    uint2 u;
    u.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
    u.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = u;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && p.lse != nullptr)
    p.lse[wid] = L > 0.f ? (M + ptx::lg2(L)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace tessera
