// The attention block's prologue on B200 (sm_100a): RMSNorm of the hidden
// states, and the rotary embedding of the projected queries and keys with the
// split into the attention layout.  The decoder of the Tessera pages is a
// transformer with RMSNorm, RoPE, grouped-query attention and SwiGLU, and its
// kernels include a fused RMSNorm; between the two steps sits the Q/K/V
// projection, a plain GEMM.
//
//   RMSNorm:  y[r,c] = x[r,c] / sqrt(mean_c x[r,c]^2 + eps) * w[c]
//   RoPE (element i paired with i + d/2, theta_i = base^(-2i/d), a = p theta_i):
//     y[i] = x[i] cos a - x[i+d/2] sin a,  y[i+d/2] = x[i] sin a + x[i+d/2] cos a
//
// Both kernels read and write each element once and do a few flops per byte:
// they are bound by HBM bandwidth.  bf16 in and out, fp32 arithmetic, angles
// in fp64 (a position of 10^5 times theta_0 = 1 keeps its fraction).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace tessera {

constexpr int kNormMaxVec = 32;  // 16-byte vectors per lane: dim <= 32 * 32 * 8 = 8192

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// A warp per row (8 rows per 256-thread CTA, rows dealt grid-stride).  The
// row stays in registers (VPT 16-byte vectors per lane, dim <= 256 * VPT)
// between the sum of squares and the scaled write.
template <int VPT>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const __nv_bfloat16* __restrict__ x,
                                                      const __nv_bfloat16* __restrict__ w,
                                                      __nv_bfloat16* y, long long rows, int dim,
                                                      float eps) {
  const int lane = threadIdx.x & 31;
  const int nvec = dim / 8;  // 16-byte vectors per row
  const float inv_dim = 1.f / static_cast<float>(dim);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * dim);
    uint4 v[VPT];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int vi = lane + 32 * j;
      if (vi < nvec) {
        v[j] = ld_stream_v4(xr + vi);
        const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf_lo(u[e]), b = bf_hi(u[e]);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(fmaf(ss, inv_dim, eps));
    uint4* yr = reinterpret_cast<uint4*>(y + r * dim);
    const uint4* wv = reinterpret_cast<const uint4*>(w);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int vi = lane + 32 * j;
      if (vi < nvec) {
        const uint4 g = wv[vi];
        const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf2(bf_lo(u[e]) * inv * bf_lo(gw[e]), bf_hi(u[e]) * inv * bf_hi(gw[e]));
        st_stream_v4(yr + vi, make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}

// Wide rows: a warp per row in two passes, 4 vectors per lane in flight per
// step: the sum of squares, then the scaled write from a second read, which
// the row's recent first read leaves in L2.  64 registers (4 CTAs, 32 warps
// per SM) instead of the 104 a 4096-wide row held in registers takes.
__global__ void __launch_bounds__(256, 4) rmsnorm_2pass_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const __nv_bfloat16* __restrict__ w,
                                                            __nv_bfloat16* y, long long rows,
                                                            int dim, float eps) {
  const int lane = threadIdx.x & 31;
  const int nvec = dim / 8;
  const float inv_dim = 1.f / static_cast<float>(dim);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * dim);
    float ss = 0.f;
    for (int v0 = lane; v0 < nvec; v0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (v0 + 32 * j < nvec) v[j] = xr[v0 + 32 * j];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (v0 + 32 * j < nvec) {
          const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = bf_lo(u[e]), b = bf_hi(u[e]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
          }
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(fmaf(ss, inv_dim, eps));
    uint4* yr = reinterpret_cast<uint4*>(y + r * dim);
    const uint4* wv = reinterpret_cast<const uint4*>(w);
    for (int v0 = lane; v0 < nvec; v0 += 128) {
      uint4 v[4], g[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (v0 + 32 * j < nvec) {
          v[j] = ld_stream_v4(xr + v0 + 32 * j);  // the last read of x: evict first
          g[j] = wv[v0 + 32 * j];
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (v0 + 32 * j < nvec) {
          const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
          const uint32_t gw[4] = {g[j].x, g[j].y, g[j].z, g[j].w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[e] = pack_bf2(bf_lo(u[e]) * inv * bf_lo(gw[e]), bf_hi(u[e]) * inv * bf_hi(gw[e]));
          st_stream_v4(yr + v0 + 32 * j, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
    }
  }
}

constexpr int kRopeTokens = 16;  // tokens per CTA
constexpr int kRopeThreads = 256;

// A CTA per (b, 16 consecutive tokens).  Thread (token tt, slot j < 16): pair
// chunk c = j % (D/16) (pairs 8c .. 8c+7, i.e. columns 8c.. and 8c+D/2..) and
// the heads h with h % HS == j / (D/16), HS = 16 / (D/16).  The thread's eight
// angles are computed once (fp64) and used for all of its query and key heads;
// its value heads are copied.  A head's rows of the 16 tokens are contiguous
// in the output, so the CTA writes runs of 16 rows.
template <int D>
__global__ void __launch_bounds__(kRopeThreads)
    rope_qkv_kernel(const __nv_bfloat16* __restrict__ qkv, const int32_t* __restrict__ positions,
                    __nv_bfloat16* q, __nv_bfloat16* k, __nv_bfloat16* v, int B, int T, int Hq,
                    int Hkv, double log2_base) {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  constexpr int P8 = D / 16;  // 8-pair chunks per head
  constexpr int HS = 16 / P8; // head classes
  const int tiles = (T + kRopeTokens - 1) / kRopeTokens;
  const int b = blockIdx.x / tiles;
  const int t = (blockIdx.x % tiles) * kRopeTokens + (threadIdx.x >> 4);
  if (b >= B || t >= T) return;
  const int j = threadIdx.x & 15;
  const int c = j % P8, hc = j / P8;
  const long long bt = static_cast<long long>(b) * T + t;
  const double pos = positions != nullptr ? static_cast<double>(positions[bt])
                                          : static_cast<double>(t);
  float cs[8], sn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int i = 8 * c + e;
    const double theta = exp2(-2.0 * i / D * log2_base);
    double s_, c_;
    sincos(pos * theta, &s_, &c_);
    cs[e] = static_cast<float>(c_);
    sn[e] = static_cast<float>(s_);
  }
  const int H3 = Hq + 2 * Hkv;
  const __nv_bfloat16* tok = qkv + bt * H3 * D;
  // the thread's heads in groups of 4, each group's loads issued together
  for (int h0 = hc; h0 < H3; h0 += 4 * HS) {
    uint4 lo4[4], hi4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = h0 + u * HS;
      if (h < H3) {
        lo4[u] = ld_stream_v4(tok + h * D + 8 * c);
        hi4[u] = ld_stream_v4(tok + h * D + D / 2 + 8 * c);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = h0 + u * HS;
      if (h >= H3) break;
      const uint4 lo = lo4[u], hi = hi4[u];
      __nv_bfloat16* dst;
      uint4 olo = lo, ohi = hi;
      if (h < Hq + Hkv) {
        const uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t bb[4] = {hi.x, hi.y, hi.z, hi.w};
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = bf_lo(a[e]), x1 = bf_hi(a[e]);      // elements i, i+1
          const float y0 = bf_lo(bb[e]), y1 = bf_hi(bb[e]);    // elements i+D/2, i+1+D/2
          const float c0 = cs[2 * e], s0 = sn[2 * e], c1 = cs[2 * e + 1], s1 = sn[2 * e + 1];
          ol[e] = pack_bf2(fmaf(x0, c0, -y0 * s0), fmaf(x1, c1, -y1 * s1));
          oh[e] = pack_bf2(fmaf(x0, s0, y0 * c0), fmaf(x1, s1, y1 * c1));
        }
        olo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        ohi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
        dst = h < Hq ? q + ((static_cast<long long>(b) * Hq + h) * T + t) * D
                     : k + ((static_cast<long long>(b) * Hkv + (h - Hq)) * T + t) * D;
      } else {
        dst = v + ((static_cast<long long>(b) * Hkv + (h - Hq - Hkv)) * T + t) * D;
      }
      st_stream_v4(dst + 8 * c, olo);
      st_stream_v4(dst + D / 2 + 8 * c, ohi);
    }
  }
}

}  // namespace tessera
