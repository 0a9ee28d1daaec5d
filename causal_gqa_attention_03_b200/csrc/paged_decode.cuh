// One decoding step of grouped-query attention over a block-paged key/value
// cache (the serving engine's paged KV cache of the Tessera pages), for B200
// (sm_100a): the parameters, the chunk stream's bookkeeping and the merge.
//
// Sequence b has seq_lens[b] cached tokens; token j lives in physical block
// block_table[b][j / bs], row j % bs.  Query head h (one query row per
// sequence) attends to all of them through key/value head h / G:
//   O[b,h,:] = sum_j softmax_j(scale * <q[b,h], k_j>) v_j,  LSE = log-sum-exp.
//
// The step reads every cached key and value once and does a few flops per
// byte, so it is bound by HBM bandwidth.  An item is one sequence and
// key/value head, for GT of its G query heads; its tokens form ceil(n / 128)
// chunks.
//   1. paged_decode_tc_kernel (paged_decode_tc.cuh), persistent (one CTA per
//      SM).  The chunks of all items, item after item, form one stream; CTA k
//      takes the k-th of gridDim.x equal contiguous shares of it, so every SM
//      moves the same number of chunks whatever the lengths.  It runs an
//      online softmax over the consecutive chunks of an item (a segment); at
//      a segment's end the unnormalised o, the running max m and the sum l go
//      to partial slot (item, k - first CTA of the item), and the CTA that
//      ends an item records its slot count.
//   2. paged_decode_merge_kernel (below): a CTA per (b, h) combines the slots:
//      M = max m_s, L = sum l_s 2^(m_s - M), O = sum o_s 2^(m_s - M) / L.
// Scores are in log2 units (q is multiplied by scale * log2(e)).
// A sequence length above the step's maximum (or negative), or a block id
// outside the cache among the pages a chunk needs, sets a device error code;
// such a sequence is empty, such a chunk contributes nothing, and nothing
// outside the cache is read.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd_sm100.cuh"

namespace tessera {

constexpr uint32_t kErrDecodeInput = 20;  // a sequence length or block id out of range
constexpr uint32_t kErrDecodeWait = 21;   // a wait of the decode pipeline gave up

constexpr int kDecodeChunk = 128;  // tokens per chunk

// flags of a ring stage
constexpr int kStageBad = 1;        // a page of the chunk is not in the cache: skip it
constexpr int kStageSegFirst = 2;   // first chunk of this CTA's segment of the item (q copied)
constexpr int kStageSegLast = 4;    // last chunk of the segment: write the partial
constexpr int kStageItemLast = 8;   // last chunk of the item: record the slot count

struct DecodeParams {
  const __nv_bfloat16* q;      // [B, Hq, D]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  __nv_bfloat16* o;            // [B, Hq, D]
  float* lse;                  // [B, Hq] or null
  float* part_o;               // [B*Hq, nslot, D]  unnormalised partial outputs
  float* part_ml;              // [B*Hq, nslot, 2]  running max (log2 units) and sum
  int* slots;                  // [B*Hkv*zgroups]   partial slots written per item
  int B, Hq, Hkv, G, bs, rows_per_box, max_blocks, num_blocks, max_seq_len, nslot, zgroups;
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

__device__ __forceinline__ int decode_chunks(int n) {
  return (n + kDecodeChunk - 1) / kDecodeChunk;
}

// Bounded wait on an mbarrier phase (no other CTA's state matters here).
__device__ __forceinline__ bool decode_wait(uint64_t* bar, uint32_t parity) {
  // a completed phase is seen by the non-blocking test (the blocking try_wait
  // costs a few hundred cycles even then)
  if (ptx::mbar_test_wait(bar, parity)) return true;
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && ptx::globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ long long warp_incl_scan(long long x, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  return x;
}

// The producer's view of one chunk of the stream.
struct DecodeCursor {
  int b, n, nchunks;  // sequence, its length and chunks
  int gz;             // g * zgroups + z
  int c;              // chunk within the item
  long long item0;    // stream position of the item's first chunk
  int slot;           // the item's partial slot written by this CTA
};

// A CTA per (b, h): warp w combines slots w, w + 8, ... (up to 8 at a time,
// loads issued together), then the warps' sums are added.  Lanes own D/32
// columns.
template <int D>
__global__ void __launch_bounds__(256) paged_decode_merge_kernel(const DecodeParams p) {
  constexpr int PER = D / 32;
  __shared__ float sred[8][D];
  __shared__ float sw[8];
  const long long wid = blockIdx.x;  // b * Hq + h
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = static_cast<int>(wid / p.Hq), h = static_cast<int>(wid % p.Hq);
  const int n = decode_len(p, b);
  int ns = 0;
  if (n > 0) {
    const int gt = p.G / p.zgroups;
    const int gz = (h / p.G) * p.zgroups + (h % p.G) / gt;
    ns = p.slots[static_cast<long long>(b) * p.Hkv * p.zgroups + gz];
    if (ns < 1 || ns > p.nslot) {  // not written by this step: cannot happen for valid input
      if (tid == 0) decode_error(p, kErrDecodeWait);
      ns = 0;
    }
  }
  const float* ml = p.part_ml + wid * p.nslot * 2;
  float M = -INFINITY;
  for (int c = tid; c < ns; c += 256) M = fmaxf(M, ml[2 * c]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) sw[warp] = M;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) M = fmaxf(M, sw[w]);
  __syncthreads();
  float L = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const float* po = p.part_o + wid * p.nslot * D + lane * PER;
  for (int c0 = warp; c0 < ns; c0 += 64) {
    float mm[8], ll[8], x[8][PER];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + 8 * j;
      mm[j] = -INFINITY;
      ll[j] = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) x[j][e] = 0.f;
      if (c < ns) {
        mm[j] = ml[2 * c];
        ll[j] = ml[2 * c + 1];
        if constexpr (PER == 4) {
          const float4 v = *reinterpret_cast<const float4*>(po + static_cast<long long>(c) * D);
          x[j][0] = v.x;
          x[j][1] = v.y;
          x[j][2] = v.z;
          x[j][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(po + static_cast<long long>(c) * D);
          x[j][0] = v.x;
          x[j][1] = v.y;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (mm[j] != -INFINITY) {  // -inf: a segment whose chunks were all dropped
        const float w = ptx::ex2(mm[j] - M);
        L = fmaf(w, ll[j], L);
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, x[j][e], acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) sred[warp][lane * PER + e] = acc[e];
  if (lane == 0) sw[warp] = L;
  __syncthreads();
  if (tid < D) {
    float o = 0.f, Lt = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      o += sred[w][tid];
      Lt += sw[w];
    }
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    p.o[wid * D + tid] = __float2bfloat16_rn(o * inv);
    if (tid == 0 && p.lse != nullptr)
      p.lse[wid] = Lt > 0.f ? (M + ptx::lg2(Lt)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace tessera
