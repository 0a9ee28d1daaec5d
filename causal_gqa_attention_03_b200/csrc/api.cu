// C ABI of the causal grouped-query attention forward (see include/tessera_attn.h).
//
// Host side: argument checks, TMA tensor maps for Q/K/V, work decomposition,
// the kernel launch on the caller's stream, and the pipelined host-buffer
// variant (copies on two library-owned streams).  Nothing here allocates
// device memory or synchronises.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "tessera_attn.h"
#include "attn_fwd_sm100.cuh"
#include "attn_bwd_sm100.cuh"
#include "paged_decode.cuh"
#include "paged_decode_tc.cuh"
#include "prologue.cuh"

namespace {

using tessera::BwdCfg;
using tessera::BwdParams;
using tessera::FwdCfg;
using tessera::FwdParams;

thread_local int g_last_launches = 0;
std::atomic<unsigned long long> g_launch_counter{1};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [planes, T, d] bf16 viewed as a 3-D tensor (d innermost); boxes of
// 64 columns x 128 rows x 1 plane with the 128-byte swizzle.  Rows at or past
// T read as zero.
bool make_map(CUtensorMap* map, const void* base, int planes, int T, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(T) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed rows [total, H, d] bf16 viewed as a 3-D tensor (d innermost, then
// head, then row); boxes of 64 columns x 1 head x 128 rows with the 128-byte
// swizzle, which land in shared memory as the same [128 rows][64] sub-tile.
// Rows at or past `total` read as zero.
bool make_map_packed(CUtensorMap* map, const void* base, int total, int H, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(total)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One launch of the forward.  With cu_seqlens (device, [B+1]) the B
// sequences are packed ([total, H, d]) and T is the longest length.
template <int D>
int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int T, int causal, float scale, cudaStream_t stream,
           const int* cu_seqlens = nullptr, int total = 0) {
  using C = FwdCfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TESSERA_ERR_CUDA;
  static std::atomic<int> sm_count[64];
  if (dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  static std::atomic<long long> l2_size[64];
  int sms = sm_count[dev].load(std::memory_order_acquire);
  long long l2_bytes = l2_size[dev].load(std::memory_order_acquire);
  if (sms == 0) {
    int l2 = 0;
    if (cudaFuncSetAttribute(tessera::attn_fwd_sm100_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || sms <= 0)
      return TESSERA_ERR_CUDA;
    l2_bytes = l2;
    l2_size[dev].store(l2_bytes, std::memory_order_release);
    sm_count[dev].store(sms, std::memory_order_release);
  }

  CUtensorMap tm_q, tm_k, tm_v;
  if (cu_seqlens != nullptr) {
    if (!make_map_packed(&tm_q, q, total, Hq, D) || !make_map_packed(&tm_k, k, total, Hkv, D) ||
        !make_map_packed(&tm_v, v, total, Hkv, D))
      return TESSERA_ERR_CUDA;
  } else if (!make_map(&tm_q, q, B * Hq, T, D) || !make_map(&tm_k, k, B * Hkv, T, D) ||
             !make_map(&tm_v, v, B * Hkv, T, D)) {
    return TESSERA_ERR_CUDA;
  }

  FwdParams p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = T;
  p.G = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.nqb = (T + C::BM - 1) / C::BM;
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  long long units;
  if (p.pair_heads) {
    p.units_per_step = B * Hkv * (p.G / 2);
    units = static_cast<long long>(p.units_per_step) * p.nqb;
  } else {
    p.units_per_step = B * Hq;
    units = static_cast<long long>(p.units_per_step) * ((p.nqb + 1) / 2);
  }
  if (units > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;
  p.num_units = static_cast<int>(units);
  // Positions r of one step: consecutive ones share a (batch, K/V head) slice.
  const int r_per_slice = p.pair_heads ? p.G / 2 : p.G;
  const int nsteps = static_cast<int>(units / p.units_per_step);
  p.r_group = p.units_per_step;
  if (cu_seqlens != nullptr) {
    p.r_group = p.units_per_step / B;  // one sequence per group
  } else {
    // When the whole K/V exceeds L2, walk groups of slices whose K/V fits in
    // half of it, each with at least two units per CTA, sizes evened out.
    const long long slice_bytes = 2LL * T * D * 2;
    const long long slices = static_cast<long long>(B) * Hkv;
    if (slices * slice_bytes > l2_bytes) {
      long long per = (l2_bytes / 2) / slice_bytes;
      const long long min_per = (2LL * sms + static_cast<long long>(r_per_slice) * nsteps - 1) /
                                (static_cast<long long>(r_per_slice) * nsteps);
      if (per < min_per) per = min_per;
      if (per < 1) per = 1;
      if (per < slices) {
        const long long groups = (slices + per - 1) / per;
        per = (slices + groups - 1) / groups;
        p.r_group = static_cast<int>(per * r_per_slice);
      }
    }
  }
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.launch_id = g_launch_counter.fetch_add(1, std::memory_order_relaxed);
  p.cu_seqlens = cu_seqlens;
  p.total = total;

  // persistent: one CTA per SM, each walking its share of the units
  const unsigned grid = static_cast<unsigned>(units < sms ? units : sms);
  tessera::attn_fwd_sm100_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tm_q, tm_k, tm_v,
                                                                                p);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  g_last_launches = 1;
  return TESSERA_OK;
}

// Checks shared by the entry points (before any CUDA call).  Returns
// TESSERA_OK with *empty set when there is nothing to compute.
int check_args(const void* q, const void* k, const void* v, const void* o, const float* lse,
               int B, int Hq, int Hkv, int T, int d, int causal, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TESSERA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return TESSERA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TESSERA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TESSERA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) {
    *empty = true;
    return TESSERA_OK;
  }
  // sizes in bytes; every product below stays far inside 64 bits for int inputs
  const size_t q_bytes = static_cast<size_t>(B) * Hq * T * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * Hkv * T * d * 2;
  const size_t lse_bytes = static_cast<size_t>(B) * Hq * T * 4;
  if (static_cast<long long>(B) * Hq > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned16(lse)))
    return TESSERA_ERR_MISALIGNED;
  if (overlaps(o, q_bytes, q, q_bytes) || overlaps(o, q_bytes, k, kv_bytes) ||
      overlaps(o, q_bytes, v, kv_bytes) || overlaps(lse, lse_bytes, q, q_bytes) ||
      overlaps(lse, lse_bytes, k, kv_bytes) || overlaps(lse, lse_bytes, v, kv_bytes) ||
      overlaps(lse, lse_bytes, o, q_bytes))
    return TESSERA_ERR_INVALID_ARG;
  return TESSERA_OK;
}

int launch_d(int d, const void* q, const void* k, const void* v, void* o, float* lse, int B,
             int Hq, int Hkv, int T, int causal, float scale, cudaStream_t s) {
  if (d == 64) return launch<64>(q, k, v, o, lse, B, Hq, Hkv, T, causal, scale, s);
  return launch<128>(q, k, v, o, lse, B, Hq, Hkv, T, causal, scale, s);
}

// Streams and events of the host-buffer pipeline, created on first use per
// device and kept for the life of the process.
// The pieces' kernels go round-robin over kPipeKernelStreams streams, so a
// piece whose inputs have arrived starts on the SMs that the previous piece's
// last (heaviest) units leave idle instead of waiting for that kernel to end.
constexpr int kPipeKernelStreams = 4;
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaStream_t run[kPipeKernelStreams] = {};
  cudaEvent_t start = nullptr, in_done = nullptr, k_done = nullptr, out_done = nullptr;
};
std::mutex g_pipe_mu;
HostPipe g_pipes[64];

// Destroys whatever a partial set-up created and clears the handles, so a
// later call starts from nothing instead of leaking the earlier objects.
void host_pipe_reset(HostPipe& h) {
  for (cudaEvent_t* e : {&h.start, &h.in_done, &h.k_done, &h.out_done}) {
    if (*e != nullptr) cudaEventDestroy(*e);
    *e = nullptr;
  }
  for (cudaStream_t* s : {&h.in, &h.out}) {
    if (*s != nullptr) cudaStreamDestroy(*s);
    *s = nullptr;
  }
  for (cudaStream_t& s : h.run) {
    if (s != nullptr) cudaStreamDestroy(s);
    s = nullptr;
  }
  h.ready = false;
}

HostPipe* host_pipe(int dev) {
  HostPipe& h = g_pipes[dev];
  if (h.ready) return &h;
  bool ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess;
  for (cudaStream_t& s : h.run)
    ok = ok && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess;
  for (cudaEvent_t* e : {&h.start, &h.in_done, &h.k_done, &h.out_done})
    ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    host_pipe_reset(h);
    return nullptr;
  }
  h.ready = true;
  return &h;
}

// Bytes of fp32 workspace the backward needs: D = rowsum(dO * O) [B,Hq,T].
size_t bwd_workspace_bytes(int B, int Hq, int T, int /*d*/) {
  return static_cast<size_t>(B) * Hq * T * 4;
}

// Parts per (batch, key/value head, key block) of the dK/dV kernel: doubled
// while the units number under 512 (about four per SM) and the group's query
// heads divide evenly, up to 8.  Depends on the shape only.
int bwd_split(int B, int Hkv, int G, int T) {
  const long long units = static_cast<long long>(B) * Hkv * ((T + 127) / 128);
  int s = 1;
  while (s < 8 && units * s < 512 && G % (2 * s) == 0) s *= 2;
  return s;
}

// Byte offset of the split partials in the workspace (after D, 256-aligned)
// and the whole workspace with them: [split][B*Hkv*T][2][d] fp32.
size_t bwd_part_offset(int B, int Hq, int T, int d) {
  return (bwd_workspace_bytes(B, Hq, T, d) + 255) & ~static_cast<size_t>(255);
}
size_t bwd_split_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int split) {
  if (split <= 1) return bwd_workspace_bytes(B, Hq, T, d);
  return bwd_part_offset(B, Hq, T, d) +
         static_cast<size_t>(split) * B * Hkv * T * static_cast<size_t>(d) * 2 * 4;
}

int sm_count(int dev) {
  static std::atomic<int> counts[64];
  int sms = counts[dev].load(std::memory_order_acquire);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
      return 0;
    counts[dev].store(sms, std::memory_order_release);
  }
  return sms;
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, float* ws, size_t ws_bytes, int B,
               int Hq, int Hkv, int T, int causal, float scale, cudaStream_t stream) {
  using C = BwdCfg<D>;
  using Q = tessera::DqCfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  static std::atomic<int> attr_set[64];
  if (attr_set[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(tessera::attn_bwd_dkdv_sm100_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(tessera::attn_bwd_dq_sm100_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Q::SMEM_BYTES) != cudaSuccess)
      return TESSERA_ERR_CUDA;
    attr_set[dev].store(1, std::memory_order_release);
  }
  const int sms = sm_count(dev);
  if (sms <= 0) return TESSERA_ERR_CUDA;
  const long long rows = static_cast<long long>(B) * Hq * T;
  const int nqb = (T + C::BM - 1) / C::BM;
  // kernel 2's units, split by query heads when the workspace holds the partials
  int split = bwd_split(B, Hkv, Hq / Hkv, T);
  if (split > 1 && ws_bytes < bwd_split_workspace_bytes(B, Hq, Hkv, T, D, split)) split = 1;
  const long long kv_units = static_cast<long long>(B) * Hkv * nqb * split;  // kernel 2
  const long long q_units = static_cast<long long>(B) * Hq * nqb;    // kernel 3
  if (q_units > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;  // before any launch
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  if (!make_map(&tm_q, q, B * Hq, T, D) || !make_map(&tm_k, k, B * Hkv, T, D) ||
      !make_map(&tm_v, v, B * Hkv, T, D) || !make_map(&tm_do, dout, B * Hq, T, D))
    return TESSERA_ERR_CUDA;
  float* dvec = ws;
  // 1. D = rowsum(dO * O)
  const long long prep_blocks = (rows + 7) / 8;  // 8 warps (rows) per block
  const unsigned pb = static_cast<unsigned>(prep_blocks < 4L * sms * 16 ? prep_blocks : 4L * sms * 16);
  tessera::attn_bwd_prep_kernel<D><<<pb, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), dvec, rows);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  BwdParams p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = T;
  p.G = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.nqb = nqb;
  p.lse = lse;
  p.dvec = dvec;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.split = split;
  // batch-major dK/dV units when one batch alone has two units per CTA
  p.kv_batch_major =
      (B > 1 && static_cast<long long>(Hkv) * split * nqb >= 2LL * sms) ? 1 : 0;
  // batch-major dQ units when one batch has two units per CTA and K/V
  // (B * Hkv * T * d, both) does not fit in L2
  int l2_bytes = 0;
  if (cudaDeviceGetAttribute(&l2_bytes, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
    return TESSERA_ERR_CUDA;
  p.q_batch_major = (B > 1 && static_cast<long long>(Hq) * nqb >= 2LL * sms &&
                     4.0 * B * Hkv * T * D > static_cast<double>(l2_bytes))
                        ? 1
                        : 0;
  p.dkv_part = split > 1 ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) +
                                                    bwd_part_offset(B, Hq, T, D))
                         : nullptr;
  // 2. dK, dV: units (batch, key/value head, key block, query-head part)
  p.num_units = static_cast<int>(kv_units);
  p.launch_id = g_launch_counter.fetch_add(1, std::memory_order_relaxed);
  const unsigned grid = static_cast<unsigned>(kv_units < sms ? kv_units : sms);
  tessera::attn_bwd_dkdv_sm100_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
      tm_q, tm_k, tm_v, tm_do, p);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  if (split > 1) {
    // 2b. dK, dV = the partials summed in part order
    const long long kv_rows = static_cast<long long>(B) * Hkv * T;
    const long long n4 = kv_rows * 2 * (D / 4);
    const long long blocks = (n4 + 255) / 256;
    const unsigned rb = static_cast<unsigned>(blocks < 8LL * sms ? blocks : 8LL * sms);
    tessera::attn_bwd_dkv_reduce_kernel<D><<<rb, 256, 0, stream>>>(
        p.dkv_part, p.dk, p.dv, kv_rows, split);
    if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  }
  // 3. dQ: units (batch, query head, query block)
  p.num_units = static_cast<int>(q_units);
  p.launch_id = g_launch_counter.fetch_add(1, std::memory_order_relaxed);
  const unsigned qgrid = static_cast<unsigned>(q_units < sms ? q_units : sms);
  tessera::attn_bwd_dq_sm100_kernel<D><<<qgrid, Q::THREADS, Q::SMEM_BYTES, stream>>>(
      tm_k, tm_v, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(dout),
      p);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  g_last_launches = split > 1 ? 4 : 3;
  return TESSERA_OK;
}

// Checks of the backward's arguments (before any CUDA call).  With
// check_ws, also the caller's workspace: non-NULL, 16-byte aligned, large
// enough, and clear of every other buffer.
int check_bwd_args(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, const void* dq, const void* dk, const void* dv,
                   const void* workspace, size_t workspace_bytes, bool check_ws, int B, int Hq,
                   int Hkv, int T, int d, int causal, float scale, bool* empty) {
  // Q/K/V and O: the forward's rules (O plays the output, LSE its LSE).
  const int st = check_args(q, k, v, o, lse, B, Hq, Hkv, T, d, causal, scale, empty);
  if (st != TESSERA_OK || *empty) return st;
  if (!lse || !dout || !dq || !dk || !dv || (check_ws && !workspace))
    return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (check_ws && !aligned16(workspace)))
    return TESSERA_ERR_MISALIGNED;
  const size_t ws_bytes = bwd_workspace_bytes(B, Hq, T, d);
  if (check_ws && workspace_bytes < ws_bytes) return TESSERA_ERR_INVALID_ARG;
  const size_t q_bytes = static_cast<size_t>(B) * Hq * T * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * Hkv * T * d * 2;
  const size_t lse_bytes = static_cast<size_t>(B) * Hq * T * 4;
  // outputs (and the workspace) must not overlap any input or each other
  const void* ins[6] = {q, k, v, o, lse, dout};
  const size_t in_bytes[6] = {q_bytes, kv_bytes, kv_bytes, q_bytes, lse_bytes, q_bytes};
  const void* outs[4] = {dq, dk, dv, check_ws ? workspace : nullptr};
  const size_t out_bytes[4] = {q_bytes, kv_bytes, kv_bytes, ws_bytes};
  for (int a = 0; a < 4; ++a) {
    for (int i = 0; i < 6; ++i)
      if (overlaps(outs[a], out_bytes[a], ins[i], in_bytes[i])) return TESSERA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b])) return TESSERA_ERR_INVALID_ARG;
  }
  return TESSERA_OK;
}

// Workspace of tessera_attn_bwd_noalloc: a device array of the library's own
// module (one per device, set up when the module loads), so that entry point
// needs no allocation.  Calls that overlap in time on one device share it.
constexpr size_t kNoAllocScratchBytes = 16ull << 20;
__device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

// Address of g_bwd_scratch on the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  static std::atomic<void*> addr[64];
  void* a = addr[dev].load(std::memory_order_acquire);
  if (a == nullptr) {
    if (cudaGetSymbolAddress(&a, g_bwd_scratch) != cudaSuccess || a == nullptr)
      return TESSERA_ERR_CUDA;
    addr[dev].store(a, std::memory_order_release);
  }
  *out = a;
  return TESSERA_OK;
}


// ------------------------------------------------------------ paged decode

// A paged cache [num_blocks, Hkv, bs, d] bf16 viewed as a 2-D tensor of
// num_blocks * Hkv * bs rows of d columns; boxes of 64 columns x box_rows
// rows with the 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, long long rows, int d, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t elem[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same cache as a 4-D tensor of 8-row atoms: (64 columns, 8 rows at 256 B,
// 2 column halves at 128 B, rows / 8 atoms at 2 KB), 128-byte swizzle; a box
// of box_rows / 8 atoms lands as [atom][half][8 rows][64 columns].  d = 128.
bool make_cache_map_atoms(CUtensorMap* map, const void* base, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, 8, 2, static_cast<cuuint64_t>(rows / 8)};
  cuuint64_t strides[3] = {256, 128, 2048};
  cuuint32_t box[4] = {64, 8, 2, static_cast<cuuint32_t>(box_rows / 8)};
  cuuint32_t elem[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

long long decode_chunks(int max_seq_len) {
  return (static_cast<long long>(max_seq_len) + tessera::kDecodeChunk - 1) / tessera::kDecodeChunk;
}

// Bytes of workspace the decode step needs: fp32 partial outputs
// [B*Hq, slots, d] and (max, sum) pairs [B*Hq, slots, 2] with one slot per
// possible 128-token chunk, then an int slot count per item (<= B*Hq items),
// rounded up to 16 bytes.
size_t decode_workspace_bytes(int B, int Hq, int max_seq_len, int d) {
  const size_t heads = static_cast<size_t>(B) * Hq;
  const size_t slots = static_cast<size_t>(decode_chunks(max_seq_len));
  if (slots == 0) return 0;
  return heads * slots * (static_cast<size_t>(d) + 2) * 4 + (heads * 4 + 15) / 16 * 16;
}

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Checks of the decode step's arguments (before any CUDA call).
int check_decode_args(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens, const void* o,
                      const float* lse, const void* workspace, size_t workspace_bytes, int B,
                      int Hq, int Hkv, int d, int bs, int max_blocks, int num_blocks,
                      int max_seq_len, float scale, bool* empty) {
  *empty = false;
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TESSERA_ERR_INVALID_ARG;
  if (max_blocks < 1 || num_blocks < 1 || max_seq_len < 0) return TESSERA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return TESSERA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TESSERA_ERR_UNSUPPORTED;
  if (!pow2(bs) || bs < 8) return TESSERA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_seq_len) > static_cast<long long>(max_blocks) * bs)
    return TESSERA_ERR_INVALID_ARG;
  // TMA row coordinates are 32-bit
  if (static_cast<long long>(num_blocks) * Hkv * bs > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;
  if (B == 0) {
    *empty = true;
    return TESSERA_OK;
  }
  const long long heads = static_cast<long long>(B) * Hq;
  const long long nch = decode_chunks(max_seq_len);
  if (heads * nch > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o) return TESSERA_ERR_INVALID_ARG;
  const size_t ws_bytes = decode_workspace_bytes(B, Hq, max_seq_len, d);
  if (ws_bytes > 0 && (!workspace || workspace_bytes < ws_bytes)) return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (ws_bytes > 0 && !aligned16(workspace)) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return TESSERA_ERR_MISALIGNED;
  const size_t q_bytes = static_cast<size_t>(heads) * d * 2;
  const size_t cache_bytes = static_cast<size_t>(num_blocks) * Hkv * bs * d * 2;
  const size_t table_bytes = static_cast<size_t>(B) * max_blocks * 4;
  const size_t lens_bytes = static_cast<size_t>(B) * 4;
  const size_t lse_bytes = static_cast<size_t>(heads) * 4;
  const void* ins[5] = {q, k_cache, v_cache, block_table, seq_lens};
  const size_t in_bytes[5] = {q_bytes, cache_bytes, cache_bytes, table_bytes, lens_bytes};
  const void* outs[3] = {o, lse, ws_bytes > 0 ? workspace : nullptr};
  const size_t out_bytes[3] = {q_bytes, lse_bytes, ws_bytes};
  for (int a = 0; a < 3; ++a) {
    for (int i = 0; i < 5; ++i)
      if (overlaps(outs[a], out_bytes[a], ins[i], in_bytes[i])) return TESSERA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 3; ++b)
      if (overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b])) return TESSERA_ERR_INVALID_ARG;
  }
  return TESSERA_OK;
}

// The tensor-core kernel, GT = the largest power of two up to 16 dividing the
// G query heads of a group: query heads per item.
template <int D, int GT>
int launch_decode_tc(const void* k_cache, const void* v_cache, tessera::DecodeParams& p,
                     cudaStream_t stream) {
  using C = tessera::DecTcCfg<D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  static std::atomic<int> attr_set[64];
  if (attr_set[dev].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(tessera::paged_decode_tc_kernel<D, GT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return TESSERA_ERR_CUDA;
    attr_set[dev].store(1, std::memory_order_release);
  }
  p.zgroups = p.G / GT;
  int launches = 0;
  if (p.nslot > 0) {
    const long long rows = static_cast<long long>(p.num_blocks) * p.Hkv * p.bs;
    CUtensorMap tm_k, tm_v, tm_q;
    const bool kv_ok = D == 128 ? make_cache_map_atoms(&tm_k, k_cache, rows, p.rows_per_box) &&
                                      make_cache_map_atoms(&tm_v, v_cache, rows, p.rows_per_box)
                                : make_cache_map(&tm_k, k_cache, rows, D, p.rows_per_box) &&
                                      make_cache_map(&tm_v, v_cache, rows, D, p.rows_per_box);
    if (!kv_ok || !make_cache_map(&tm_q, p.q, static_cast<long long>(p.B) * p.Hq, D, GT))
      return TESSERA_ERR_CUDA;
    const int sms = sm_count(dev);
    if (sms <= 0) return TESSERA_ERR_CUDA;
    tessera::paged_decode_tc_kernel<D, GT><<<static_cast<unsigned>(sms), tessera::kDecTcThreads,
                                             C::SMEM, stream>>>(tm_k, tm_v, tm_q, p);
    if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
    ++launches;
  }
  const long long heads = static_cast<long long>(p.B) * p.Hq;  // one merge CTA each
  tessera::paged_decode_merge_kernel<D><<<static_cast<unsigned>(heads), 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  g_last_launches = launches + 1;
  return TESSERA_OK;
}

template <int D>
int launch_decode_tc_d(const void* k_cache, const void* v_cache, tessera::DecodeParams& p,
                       cudaStream_t stream) {
  const int G = p.G;
  if (G % 16 == 0) return launch_decode_tc<D, 16>(k_cache, v_cache, p, stream);
  if (G % 8 == 0) return launch_decode_tc<D, 8>(k_cache, v_cache, p, stream);
  if (G % 4 == 0) return launch_decode_tc<D, 4>(k_cache, v_cache, p, stream);
  if (G % 2 == 0) return launch_decode_tc<D, 2>(k_cache, v_cache, p, stream);
  return launch_decode_tc<D, 1>(k_cache, v_cache, p, stream);
}

}  // namespace

extern "C" int tessera_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int T, int d, int causal, float scale,
                                tessera_stream_t stream) {
  g_last_launches = 0;
  bool empty = false;
  const int st = check_args(q, k, v, o, lse, B, Hq, Hkv, T, d, causal, scale, &empty);
  if (st != TESSERA_OK || empty) return st;
  return launch_d(d, q, k, v, o, lse, B, Hq, Hkv, T, causal, scale,
                  reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int tessera_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                       float* lse, const int32_t* cu_seqlens, int B, int total,
                                       int max_seqlen, int Hq, int Hkv, int d, int causal,
                                       float scale, tessera_stream_t stream) {
  g_last_launches = 0;
  if (B < 0 || total < 0 || max_seqlen < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return TESSERA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return TESSERA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TESSERA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TESSERA_ERR_UNSUPPORTED;
  if (max_seqlen > total) return TESSERA_ERR_INVALID_ARG;
  if (B == 0 || total == 0 || max_seqlen == 0) return TESSERA_OK;
  if (!q || !k || !v || !o || !cu_seqlens) return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return TESSERA_ERR_MISALIGNED;
  const size_t q_bytes = static_cast<size_t>(total) * Hq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(total) * Hkv * d * 2;
  const size_t lse_bytes = static_cast<size_t>(total) * Hq * 4;
  const size_t cu_bytes = (static_cast<size_t>(B) + 1) * 4;
  const void* ins[4] = {q, k, v, cu_seqlens};
  const size_t in_bytes[4] = {q_bytes, kv_bytes, kv_bytes, cu_bytes};
  for (int i = 0; i < 4; ++i)
    if (overlaps(o, q_bytes, ins[i], in_bytes[i]) || overlaps(lse, lse_bytes, ins[i], in_bytes[i]))
      return TESSERA_ERR_INVALID_ARG;
  if (overlaps(o, q_bytes, lse, lse_bytes)) return TESSERA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int* cu = reinterpret_cast<const int*>(cu_seqlens);
  if (d == 64)
    return launch<64>(q, k, v, o, lse, B, Hq, Hkv, max_seqlen, causal, scale, s, cu, total);
  return launch<128>(q, k, v, o, lse, B, Hq, Hkv, max_seqlen, causal, scale, s, cu, total);
}

// One piece of the host-buffer pipeline: whole slices [s0, s1) (h0 = 0,
// h1 = G), or query heads [h0, h1) of the one slice s0 (s1 = s0 + 1).
struct HostPiece {
  int s0, s1, h0, h1;
};

// `target` pieces: contiguous ranges of whole slices while target <= slices;
// otherwise every slice cut into `split` runs of G/split query heads (split
// the smallest divisor of G that is at least ceil(target / slices), else G).
void plan_even(int slices, int G, int target, std::vector<HostPiece>& out) {
  if (target <= slices) {
    for (int c = 0; c < target; ++c) {
      const int s0 = static_cast<int>(static_cast<long long>(slices) * c / target);
      const int s1 = static_cast<int>(static_cast<long long>(slices) * (c + 1) / target);
      if (s1 > s0) out.push_back({s0, s1, 0, G});
    }
    return;
  }
  const int want = (target + slices - 1) / slices;
  int split = G;
  for (int s_ = want; s_ < G; ++s_)
    if (G % s_ == 0) {
      split = s_;
      break;
    }
  for (int sl = 0; sl < slices; ++sl)
    for (int r = 0; r < split; ++r)
      out.push_back({sl, sl + 1, r * (G / split), (r + 1) * (G / split)});
}

// The pieces of tessera_attn_fwd_host, in queue order.  chunks > 0: the even
// plan above.  chunks == 0: the even plan for 8 pieces with its last piece
// tapered: its whole slices but the last stay one piece, and the last slice's
// final min(G, 4) query heads become one piece each (the rest of that slice
// one piece before them).  The pipeline ends with the last piece's kernel and
// download, so one-head last pieces shorten that drain.
std::vector<HostPiece> plan_host_pieces(int slices, int G, int chunks) {
  std::vector<HostPiece> out;
  plan_even(slices, G, chunks > 0 ? chunks : 8, out);
  if (chunks > 0 || out.empty()) return out;
  const HostPiece last = out.back();
  out.pop_back();
  const int sl = last.s1 - 1;
  if (last.s1 - last.s0 > 1) out.push_back({last.s0, sl, 0, G});
  const int tail = (last.h1 - last.h0) < 4 ? (last.h1 - last.h0) : 4;
  if (last.h1 - tail > last.h0) out.push_back({sl, sl + 1, last.h0, last.h1 - tail});
  for (int h = last.h1 - tail; h < last.h1; ++h) out.push_back({sl, sl + 1, h, h + 1});
  return out;
}

extern "C" int tessera_attn_fwd_host_plan(int B, int Hq, int Hkv, int chunks, int* pieces,
                                          int max_pieces) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || chunks < 0 || max_pieces < 0 ||
      (max_pieces > 0 && pieces == nullptr) || static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return -TESSERA_ERR_INVALID_ARG;
  std::vector<HostPiece> plan;
  try {
    plan = plan_host_pieces(static_cast<int>(static_cast<long long>(B) * Hkv), Hq / Hkv, chunks);
  } catch (...) {
    return -TESSERA_ERR_INVALID_ARG;
  }
  const int n = static_cast<int>(plan.size());
  for (int i = 0; i < n && i < max_pieces; ++i) {
    pieces[4 * i + 0] = plan[i].s0;
    pieces[4 * i + 1] = plan[i].s1;
    pieces[4 * i + 2] = plan[i].h0;
    pieces[4 * i + 3] = plan[i].h1;
  }
  return n;
}

extern "C" int tessera_attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                                     float* lse_h, void* q_d, void* k_d, void* v_d, void* o_d,
                                     float* lse_d, int B, int Hq, int Hkv, int T, int d,
                                     int causal, float scale, int chunks,
                                     tessera_stream_t stream) {
  g_last_launches = 0;
  bool empty = false;
  const int st = check_args(q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, T, d, causal, scale, &empty);
  if (st != TESSERA_OK) return st;
  if ((lse_h == nullptr) != (lse_d == nullptr) || chunks < 0) return TESSERA_ERR_INVALID_ARG;
  if (empty) return TESSERA_OK;
  if (!q_h || !k_h || !v_h || !o_h) return TESSERA_ERR_INVALID_ARG;
  const int slices = static_cast<int>(static_cast<long long>(B) * Hkv);
  const int G = Hq / Hkv;
  std::vector<HostPiece> pieces;
  try {
    pieces = plan_host_pieces(slices, G, chunks);
  } catch (...) {  // no host memory for the plan (one entry per piece, at most B*Hq)
    return TESSERA_ERR_INVALID_ARG;
  }
  const int n_pieces = static_cast<int>(pieces.size());
  const size_t kv_slice = static_cast<size_t>(T) * d * 2;   // bytes of one K (or V) head
  const size_t q_head = kv_slice;                           // bytes of one Q (or O) head
  const size_t lse_head = static_cast<size_t>(T) * 4;       // bytes of one head's LSE rows
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = host_pipe(dev);
  if (!hp) return TESSERA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Everything queued on `stream` before this call (readers or writers of the
  // staging buffers) comes first.
  if (cudaEventRecord(hp->start, s) != cudaSuccess ||
      cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return TESSERA_ERR_CUDA;
  const auto c8 = [](const void* p, size_t off) { return static_cast<const char*>(p) + off; };
  const auto m8 = [](void* p, size_t off) { return static_cast<char*>(p) + off; };
  int launches = 0;
  for (int c = 0; c < n_pieces; ++c) {
    const int s0 = pieces[c].s0, s1 = pieces[c].s1, h0 = pieces[c].h0, h1 = pieces[c].h1;
    const int n = s1 - s0;
    const bool whole = (h0 == 0 && h1 == G);
    const int nq = whole ? n * G : h1 - h0;  // query heads of the launch
    const size_t qo = q_head * (static_cast<size_t>(s0) * G + h0);
    const size_t lo = lse_head * (static_cast<size_t>(s0) * G + h0);
    const size_t ko = kv_slice * s0;
    if (h0 == 0 &&
        (cudaMemcpyAsync(m8(k_d, ko), c8(k_h, ko), kv_slice * n, cudaMemcpyHostToDevice, hp->in) !=
             cudaSuccess ||
         cudaMemcpyAsync(m8(v_d, ko), c8(v_h, ko), kv_slice * n, cudaMemcpyHostToDevice, hp->in) !=
             cudaSuccess))
      return TESSERA_ERR_CUDA;
    cudaStream_t run = hp->run[launches % kPipeKernelStreams];
    if (cudaMemcpyAsync(m8(q_d, qo), c8(q_h, qo), q_head * nq, cudaMemcpyHostToDevice, hp->in) !=
            cudaSuccess ||
        cudaEventRecord(hp->in_done, hp->in) != cudaSuccess ||
        cudaStreamWaitEvent(run, hp->in_done, 0) != cudaSuccess)
      return TESSERA_ERR_CUDA;
    const int lst = launch_d(d, m8(q_d, qo), m8(k_d, ko), m8(v_d, ko), m8(o_d, qo),
                             lse_d ? reinterpret_cast<float*>(m8(lse_d, lo)) : nullptr, 1, nq, n,
                             T, causal, scale, run);
    if (lst != TESSERA_OK) return lst;
    ++launches;
    if (cudaEventRecord(hp->k_done, run) != cudaSuccess ||
        cudaStreamWaitEvent(hp->out, hp->k_done, 0) != cudaSuccess ||
        cudaMemcpyAsync(m8(o_h, qo), c8(o_d, qo), q_head * nq, cudaMemcpyDeviceToHost, hp->out) !=
            cudaSuccess)
      return TESSERA_ERR_CUDA;
    if (lse_h && cudaMemcpyAsync(m8(lse_h, lo), c8(lse_d, lo), lse_head * nq,
                                 cudaMemcpyDeviceToHost, hp->out) != cudaSuccess)
      return TESSERA_ERR_CUDA;
  }
  // Work queued on `stream` after this call sees the host outputs complete.
  if (cudaEventRecord(hp->out_done, hp->out) != cudaSuccess ||
      cudaStreamWaitEvent(s, hp->out_done, 0) != cudaSuccess)
    return TESSERA_ERR_CUDA;
  g_last_launches = launches;
  return TESSERA_OK;
}

extern "C" size_t tessera_attn_bwd_workspace_bytes(int B, int Hq, int T, int d) {
  if (B < 0 || Hq < 1 || T < 0 || (d != 64 && d != 128)) return 0;
  return bwd_workspace_bytes(B, Hq, T, d);
}

extern "C" int tessera_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                                int T, int d, int causal, float scale, tessera_stream_t stream) {
  g_last_launches = 0;
  bool empty = false;
  const int st = check_bwd_args(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                true, B, Hq, Hkv, T, d, causal, scale, &empty);
  if (st != TESSERA_OK || empty) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  if (d == 64) return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, ws, workspace_bytes, B, Hq,
                                     Hkv, T, causal, scale, s);
  return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, ws, workspace_bytes, B, Hq, Hkv, T,
                         causal, scale, s);
}

extern "C" size_t tessera_attn_bwd_workspace_bytes_kv(int B, int Hq, int Hkv, int T, int d) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || T < 0 || (d != 64 && d != 128)) return 0;
  return bwd_split_workspace_bytes(B, Hq, Hkv, T, d, bwd_split(B, Hkv, Hq / Hkv, T));
}

extern "C" size_t tessera_attn_bwd_noalloc_max_workspace_bytes(void) {
  return kNoAllocScratchBytes;
}

extern "C" int tessera_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                        const void* o, const float* lse, const void* dout,
                                        void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                        int T, int d, int causal, float scale,
                                        tessera_stream_t stream) {
  g_last_launches = 0;
  bool empty = false;
  const int st = check_bwd_args(q, k, v, o, lse, dout, dq, dk, dv, nullptr, 0, false, B, Hq, Hkv,
                                T, d, causal, scale, &empty);
  if (st != TESSERA_OK || empty) return st;
  if (bwd_workspace_bytes(B, Hq, T, d) > kNoAllocScratchBytes) return TESSERA_ERR_TOO_LARGE;
  void* ws = nullptr;
  const int sst = noalloc_scratch(&ws);
  if (sst != TESSERA_OK) return sst;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* wsf = static_cast<float*>(ws);
  if (d == 64) return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, wsf, kNoAllocScratchBytes,
                                     B, Hq, Hkv, T, causal, scale, s);
  return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, wsf, kNoAllocScratchBytes, B, Hq, Hkv,
                         T, causal, scale, s);
}

extern "C" size_t tessera_attn_decode_workspace_bytes(int B, int Hq, int max_seq_len, int d) {
  if (B < 0 || Hq < 1 || max_seq_len < 0 || (d != 64 && d != 128)) return 0;
  return decode_workspace_bytes(B, Hq, max_seq_len, d);
}

extern "C" int tessera_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_table, const int32_t* seq_lens, void* o,
                                   float* lse, void* workspace, size_t workspace_bytes, int B,
                                   int Hq, int Hkv, int d, int block_size, int max_blocks,
                                   int num_blocks, int max_seq_len, float scale,
                                   tessera_stream_t stream) {
  g_last_launches = 0;
  bool empty = false;
  const int st = check_decode_args(q, k_cache, v_cache, block_table, seq_lens, o, lse, workspace,
                                   workspace_bytes, B, Hq, Hkv, d, block_size, max_blocks,
                                   num_blocks, max_seq_len, scale, &empty);
  if (st != TESSERA_OK || empty) return st;
  tessera::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.bs = block_size;
  p.rows_per_box = block_size < tessera::kDecodeChunk ? block_size : tessera::kDecodeChunk;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.max_seq_len = max_seq_len;
  p.nslot = static_cast<int>(decode_chunks(max_seq_len));
  p.zgroups = 1;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  float* ws = static_cast<float*>(workspace);
  p.part_o = ws;
  const size_t heads_slots = static_cast<size_t>(B) * Hq * p.nslot;
  p.part_ml = ws ? ws + heads_slots * d : nullptr;
  p.slots = ws ? reinterpret_cast<int*>(ws + heads_slots * (d + 2)) : nullptr;
  p.launch_id = g_launch_counter.fetch_add(1, std::memory_order_relaxed);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) return launch_decode_tc_d<64>(k_cache, v_cache, p, s);
  return launch_decode_tc_d<128>(k_cache, v_cache, p, s);
}

extern "C" int tessera_rmsnorm(const void* x, const void* w, void* y, int rows, int dim,
                               float eps, tessera_stream_t stream) {
  g_last_launches = 0;
  if (rows < 0 || dim < 1 || !(eps >= 0.f) || !std::isfinite(eps)) return TESSERA_ERR_INVALID_ARG;
  if (dim % 8 != 0 || dim > tessera::kNormMaxVec * 32 * 8) return TESSERA_ERR_UNSUPPORTED;
  if (rows == 0) return TESSERA_OK;
  if (!x || !w || !y) return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return TESSERA_ERR_MISALIGNED;
  const size_t bytes = static_cast<size_t>(rows) * dim * 2;
  // in place (y == x) is allowed; any other overlap is not
  if ((y != x && overlaps(y, bytes, x, bytes)) || overlaps(y, bytes, w, static_cast<size_t>(dim) * 2))
    return TESSERA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TESSERA_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return TESSERA_ERR_CUDA;
  const long long blocks = (static_cast<long long>(rows) + 7) / 8;  // a warp per row
  const long long cap = static_cast<long long>(sms) * 32;  // beyond residency: the scheduler balances
  const unsigned grid = static_cast<unsigned>(blocks < cap ? blocks : cap);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  const int vpt = (dim / 8 + 31) / 32;  // 16-byte vectors per lane
  if (vpt <= 4)
    tessera::rmsnorm_kernel<4><<<grid, 256, 0, s>>>(xb, wb, yb, rows, dim, eps);
  else if (vpt <= 8)
    tessera::rmsnorm_kernel<8><<<grid, 256, 0, s>>>(xb, wb, yb, rows, dim, eps);
  else  // wider rows: two passes, the second from L2
    tessera::rmsnorm_2pass_kernel<<<grid, 256, 0, s>>>(xb, wb, yb, rows, dim, eps);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  g_last_launches = 1;
  return TESSERA_OK;
}

extern "C" int tessera_rope_qkv(const void* qkv, const int32_t* positions, void* q, void* k,
                                void* v, int B, int T, int Hq, int Hkv, int d, float base,
                                tessera_stream_t stream) {
  g_last_launches = 0;
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TESSERA_ERR_INVALID_ARG;
  if (!(base > 0.f) || !std::isfinite(base)) return TESSERA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TESSERA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return TESSERA_OK;
  if (!qkv || !q || !k || !v) return TESSERA_ERR_INVALID_ARG;
  if (!aligned16(qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(positions) & 3u))
    return TESSERA_ERR_MISALIGNED;
  const long long tokens = static_cast<long long>(B) * T;
  const long long tiles = (static_cast<long long>(T) + tessera::kRopeTokens - 1) / tessera::kRopeTokens;
  if (B * tiles > 0x7fffffffLL) return TESSERA_ERR_INVALID_ARG;
  const size_t in_bytes = static_cast<size_t>(tokens) * (Hq + 2 * Hkv) * d * 2;
  const size_t q_bytes = static_cast<size_t>(tokens) * Hq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(tokens) * Hkv * d * 2;
  const size_t pos_bytes = positions ? static_cast<size_t>(tokens) * 4 : 0;
  const void* outs[3] = {q, k, v};
  const size_t out_bytes[3] = {q_bytes, kv_bytes, kv_bytes};
  for (int a = 0; a < 3; ++a) {
    if (overlaps(outs[a], out_bytes[a], qkv, in_bytes) ||
        overlaps(outs[a], out_bytes[a], positions, pos_bytes))
      return TESSERA_ERR_INVALID_ARG;
    for (int b2 = a + 1; b2 < 3; ++b2)
      if (overlaps(outs[a], out_bytes[a], outs[b2], out_bytes[b2])) return TESSERA_ERR_INVALID_ARG;
  }
  const double log2_base = std::log2(static_cast<double>(base));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(B * tiles);
  if (d == 64)
    tessera::rope_qkv_kernel<64><<<grid, tessera::kRopeThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(qkv), positions, static_cast<__nv_bfloat16*>(q),
        static_cast<__nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(v), B, T, Hq, Hkv, log2_base);
  else
    tessera::rope_qkv_kernel<128><<<grid, tessera::kRopeThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(qkv), positions, static_cast<__nv_bfloat16*>(q),
        static_cast<__nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(v), B, T, Hq, Hkv, log2_base);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  g_last_launches = 1;
  return TESSERA_OK;
}

extern "C" int tessera_attn_device_error(int* code) {
  if (!code) return TESSERA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return TESSERA_ERR_CUDA;
  unsigned long long w = 0;
  if (cudaMemcpyFromSymbol(&w, tessera::g_tessera_err, sizeof(w)) != cudaSuccess)
    return TESSERA_ERR_CUDA;
  const unsigned long long zero = 0;
  if (cudaMemcpyToSymbol(tessera::g_tessera_err, &zero, sizeof(zero)) != cudaSuccess)
    return TESSERA_ERR_CUDA;
  *code = static_cast<int>(w & 0xffffffffull);
  return TESSERA_OK;
}

extern "C" int tessera_attn_selftest_timeout(unsigned int limit_us, tessera_stream_t stream) {
  if (limit_us == 0 || limit_us > 10000000u) return TESSERA_ERR_INVALID_ARG;
  const unsigned long long id = g_launch_counter.fetch_add(1, std::memory_order_relaxed);
  tessera::attn_selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      id, static_cast<uint64_t>(limit_us) * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return TESSERA_ERR_CUDA;
  return TESSERA_OK;
}

extern "C" const char* tessera_status_str(int status) {
  switch (status) {
    case TESSERA_OK: return "ok";
    case TESSERA_ERR_INVALID_ARG: return "invalid argument";
    case TESSERA_ERR_UNSUPPORTED:
      return "unsupported head dimension (64 or 128) or block size (a power of two >= 8)";
    case TESSERA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case TESSERA_ERR_CUDA: return "CUDA runtime error";
    case TESSERA_ERR_TIMEOUT: return "device-side wait timed out";
    case TESSERA_ERR_TOO_LARGE: return "workspace needed exceeds the static scratch array";
    default: return "unknown status";
  }
}

extern "C" int tessera_attn_last_launch_count(void) { return g_last_launches; }
