/*
 * tessera_attn.h -- C ABI of the causal grouped-query FlashAttention forward
 * pass for NVIDIA B200 (sm_100a).
 *
 * The operation is the attention forward kernel that the Tessera pages name:
 * "a FlashAttention forward kernel with online softmax, causal masking,
 * grouped-query attention" (hysenlabs.com Tessera review, section "The kernel
 * set and its torch fallback"; Tessera README, "What's in it" / "Kernels"),
 * used by the decoder with "RMSNorm, RoPE, grouped-query attention and
 * SwiGLU" (Tessera README, "What's in it" / "Training side").  The pages give
 * no formula; the plain reading adopted here is scaled-dot-product attention:
 *
 *   G = Hq / Hkv; query head h reads key/value head floor(h / G)
 *   s_ij = scale * dot(Q[b,h,i,:], K[b,g,j,:]),  j <= i when causal
 *   O[b,h,i,:] = sum_j softmax_j(s_i) * V[b,g,j,:]
 *   LSE[b,h,i] = ln sum_j exp(s_ij)     (natural log of the scaled logits)
 *
 * No C++ or CUDA types appear in this header; the library links the CUDA
 * runtime statically and needs a CUDA driver only when a function below that
 * launches work is called.
 */
#ifndef TESSERA_ATTN_H
#define TESSERA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL means the legacy default stream. */
typedef struct CUstream_st *tessera_stream_t;

typedef enum {
    TESSERA_OK = 0,
    TESSERA_ERR_INVALID_ARG = 1, /* bad size, null pointer, aliasing, bad scale */
    TESSERA_ERR_UNSUPPORTED = 2, /* head dim not 64/128; decode block size; norm width */
    TESSERA_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned */
    TESSERA_ERR_CUDA = 4,        /* the CUDA runtime reported an error */
    TESSERA_ERR_TIMEOUT = 5,     /* a device-side wait gave up (see below) */
    TESSERA_ERR_TOO_LARGE = 6    /* tessera_attn_bwd_noalloc: problem over its scratch size */
} tessera_status;

/*
 * Causal (or full) grouped-query attention forward on one GPU.
 *
 * q    bf16 [B, Hq,  T, d]  device memory, contiguous row-major, read only
 * k    bf16 [B, Hkv, T, d]  device memory, contiguous row-major, read only
 * v    bf16 [B, Hkv, T, d]  device memory, contiguous row-major, read only
 * o    bf16 [B, Hq,  T, d]  device memory, written (rounded to nearest even)
 * lse  fp32 [B, Hq,  T]     device memory, written; may be NULL to skip it
 * B, Hq, Hkv, T  sizes; B >= 0, T >= 0 (either 0 returns TESSERA_OK and
 *      launches nothing), Hq >= 1, Hkv >= 1, Hq % Hkv == 0
 * d    head dimension: 64 or 128, else TESSERA_ERR_UNSUPPORTED
 * causal  1: row i attends to keys j <= i; 0: to every key j < T
 * scale   positive finite multiplier of Q.K^T (typically 1/sqrt(d))
 * stream  the CUDA stream the work is queued on
 *
 * All buffers are owned by the caller.  The call allocates no device memory,
 * does not synchronise, and returns as soon as the kernel is queued.  Every
 * pointer must be 16-byte aligned (TESSERA_ERR_MISALIGNED), non-NULL when its
 * tensor is non-empty, and o / lse must not overlap q, k, v or each other
 * (TESSERA_ERR_INVALID_ARG).  Arguments are checked before any CUDA call, so a
 * rejected call has no effect.  Launch failures return TESSERA_ERR_CUDA.
 *
 * Every wait inside the kernel is bounded; if one gives up (it never does in
 * a correct run) the kernel records the fact in a device-side error word and
 * exits without hanging.  tessera_attn_device_error() reads that word.
 */
int tessera_attn_fwd(const void *q, const void *k, const void *v, void *o,
                     float *lse, int B, int Hq, int Hkv, int T, int d,
                     int causal, float scale, tessera_stream_t stream);

/*
 * Variable-length forward: B sequences of different lengths packed into one
 * batch, each attending only to itself.  The pages' forward has a causal flag
 * (hysenlabs.com review, "The kernel set and its torch fallback"); running it
 * over a batch of mixed lengths without padding is the variant adopted here,
 * with the same per-sequence definition as tessera_attn_fwd:
 *
 *   sequence b holds rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of every tensor;
 *   with T_b its length and i, j rows of sequence b, O and LSE of row i are
 *   tessera_attn_fwd's over keys j <= i (causal) or all j < T_b.
 *
 * q           bf16 [total, Hq, d]  device, read only (token-major, packed)
 * k, v        bf16 [total, Hkv, d] device, read only
 * o           bf16 [total, Hq, d]  device, written
 * lse         fp32 [Hq, total]     device, written; may be NULL
 * cu_seqlens  int32 [B + 1] device: 0 = cu[0] <= cu[1] <= ... <= cu[B] = total
 * B >= 0, total >= 0, max_seqlen: a bound on every length, 0 .. total (it
 *             sizes the launch); B, total or max_seqlen 0 launches nothing
 * Hq, Hkv, d, causal, scale, stream  as in tessera_attn_fwd
 *
 * Checks as in tessera_attn_fwd before any CUDA call, plus cu_seqlens
 * non-NULL and 4-byte aligned and o/lse clear of every input.  The offsets
 * live on the device and are checked by the kernel: a sequence whose bounds
 * are out of order, past `total` or longer than max_seqlen is skipped (its
 * rows of o and lse are left as they were) and TESSERA_DEVICE_ERR_VARLEN_INPUT
 * is recorded for tessera_attn_device_error(); the other sequences are
 * computed as usual and nothing outside the buffers is read.  One launch.
 */
#define TESSERA_DEVICE_ERR_VARLEN_INPUT 10
int tessera_attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                            const int32_t *cu_seqlens, int B, int total, int max_seqlen,
                            int Hq, int Hkv, int d, int causal, float scale,
                            tessera_stream_t stream);

/*
 * Backward of tessera_attn_fwd: the gradients dQ, dK, dV of a loss given
 * dO = dLoss/dO, treating LSE as saved state.  The pages list the attention
 * backward as not yet built (it is the first extension after the forward);
 * the operation is the exact derivative of the forward above:
 *
 *   P_ij = exp(s_ij - LSE[b,h,i]),  D_i = <dO[b,h,i,:], O[b,h,i,:]>
 *   dS_ij = P_ij * (<dO[b,h,i,:], V[b,g,j,:]> - D_i)
 *   dQ[b,h,i,:] = scale * sum_j dS_ij K[b,g,j,:]
 *   dK[b,g,j,:] = scale * sum_{h in g, i} dS_ij Q[b,h,i,:]
 *   dV[b,g,j,:] = sum_{h in g, i} P_ij dO[b,h,i,:]
 *
 * q, k, v, o, lse  the forward's inputs and outputs (o and lse as written by
 *                  tessera_attn_fwd with the same arguments), device memory
 * dout             bf16 [B, Hq, T, d] device, read only
 * dq               bf16 [B, Hq, T, d] device, written
 * dk, dv           bf16 [B, Hkv, T, d] device, written
 * workspace        device memory of at least
 *                  tessera_attn_bwd_workspace_bytes(B, Hq, T, d) bytes
 *                  (B*Hq*T fp32: D), 16-byte aligned, owned by the caller;
 *                  overwritten (no contents need to be set before the call);
 *                  workspace_bytes gives its size.  With at least
 *                  tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)
 *                  bytes, shapes with few key/value units also get the
 *                  balanced form below.
 * other arguments  as in tessera_attn_fwd
 *
 * Checks as in tessera_attn_fwd, plus: every pointer non-NULL (lse too) and
 * 16-byte aligned, a large enough workspace, and no overlap between
 * dq/dk/dv/workspace and any input or each other.  Queues three kernels on
 * `stream` (tessera_attn_last_launch_count() = 3): D, then dK/dV (key blocks
 * as units), then dQ (query blocks as units, S and dP recomputed); no
 * atomics, so the result does not depend on scheduling.  Bounded waits as in
 * the forward.
 *
 * Balanced form (the pages have no counterpart; this is a scheduling choice
 * of this library).  When B * Hkv * ceil(T/128) is under 512 (about four
 * units per SM: multi-query attention, few batches) and the workspace holds
 * them, the dK/dV units are cut by query heads into split = 2, 4 or 8 parts
 * (G / split heads each); each part writes fp32 partial dK, dV into the
 * workspace and a fourth kernel sums them in part order into bf16
 * (tessera_attn_last_launch_count() = 4).  The split depends on the shape
 * and the workspace size only, so the result still does not depend on
 * scheduling; it differs from the three-kernel form only in the rounding of
 * the dK/dV sums.
 */
size_t tessera_attn_bwd_workspace_bytes(int B, int Hq, int T, int d);

/*
 * Workspace bytes with which tessera_attn_bwd uses its balanced form for this
 * shape: tessera_attn_bwd_workspace_bytes(B, Hq, T, d) when the shape has
 * enough key/value units, else D (256-byte aligned) followed by
 * split * B * Hkv * T * d * 2 fp32 partials.  0 for invalid sizes.
 */
size_t tessera_attn_bwd_workspace_bytes_kv(int B, int Hq, int Hkv, int T, int d);
int tessera_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                     const float *lse, const void *dout, void *dq, void *dk, void *dv,
                     void *workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                     int T, int d, int causal, float scale, tessera_stream_t stream);

/*
 * tessera_attn_bwd without a caller-supplied workspace.  (The pages have no
 * counterpart: this is an interface of this library.)  The workspace is a
 * device array in the library itself, of
 * tessera_attn_bwd_noalloc_max_workspace_bytes() bytes (16 MiB) on every
 * device the library runs on; the call allocates nothing and calls no
 * allocating routine.  Nothing in the array needs to start at zero: each call
 * sets all it reads.  Arguments, checks and results are those of
 * tessera_attn_bwd; a problem whose workspace
 * (tessera_attn_bwd_workspace_bytes) exceeds the array returns
 * TESSERA_ERR_TOO_LARGE before any CUDA call.  The balanced form is used
 * when tessera_attn_bwd_workspace_bytes_kv fits in the array.  Calls whose work overlaps in
 * time on one device (other streams or threads) share the array and race:
 * queue them on one stream.
 */
size_t tessera_attn_bwd_noalloc_max_workspace_bytes(void);
int tessera_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                             const float *lse, const void *dout, void *dq, void *dk,
                             void *dv, int B, int Hq, int Hkv, int T, int d, int causal,
                             float scale, tessera_stream_t stream);

/*
 * The same operation on host buffers, pipelined over the host link.  (The
 * pages describe the kernel only; this transfer pipeline is this library's.)
 * The problem is cut into pieces along the B*Hkv (batch, key/value head)
 * slices: a piece is a range of whole slices, or a run of query heads of one
 * slice (the slice's K/V go with its first run).  With `chunks` > 0 the plan
 * is even: `chunks` contiguous ranges of whole slices, or, when `chunks`
 * exceeds B*Hkv, every slice cut into `split` runs of G/split query heads
 * (split = the smallest divisor of G that is at least ceil(chunks / (B*Hkv)),
 * else G).  With `chunks` = 0 the plan is the even one for 8 with its last
 * piece tapered: that piece's whole slices but the last stay one piece, and
 * the last slice's final min(G', 4) query heads (G' the heads of that piece
 * within the slice) become one piece each, the rest of them one piece before.
 * tessera_attn_fwd_host_plan lists the pieces.  For each piece Q (and K/V)
 * are copied host -> device, the kernel of tessera_attn_fwd runs on it, and
 * O/LSE are copied device -> host.  Copies run on two streams and the kernels
 * round-robin on four more that the library creates per device on first use
 * (kept for the life of the process), so one piece's copies overlap the
 * others' kernels and copies, and a piece's kernel starts on the SMs the
 * previous piece's last units leave idle.
 *
 * q_h, k_h, v_h  host inputs, layouts as in tessera_attn_fwd.  Page-locked
 *                memory (cudaHostAlloc / cudaHostRegister) lets the copies
 *                overlap; pageable memory gives the same results, serialised.
 * o_h, lse_h     host outputs; lse_h may be NULL (then lse_d must be NULL).
 * q_d .. lse_d   device buffers of the full sizes, owned by the caller, with
 *                the rules of tessera_attn_fwd; they also hold the results.
 * chunks         0: the tapered plan; > 0: the even plan, as above.  Every
 *                plan gives the same bits as one tessera_attn_fwd.
 * stream         the host outputs are complete once the work queued on
 *                `stream` before the call returns has finished plus this
 *                call's work: synchronise `stream` before reading them.
 *
 * Arguments are checked as in tessera_attn_fwd (plus non-NULL host pointers
 * and chunks >= 0) before any CUDA call.  Calls are serialised by a mutex.
 * tessera_attn_last_launch_count() then reports the number of launches (one
 * per piece).
 */
int tessera_attn_fwd_host(const void *q_h, const void *k_h, const void *v_h, void *o_h,
                          float *lse_h, void *q_d, void *k_d, void *v_d, void *o_d,
                          float *lse_d, int B, int Hq, int Hkv, int T, int d, int causal,
                          float scale, int chunks, tessera_stream_t stream);

/*
 * The pieces tessera_attn_fwd_host cuts a [B, Hq | Hkv, T, d] problem into for
 * `chunks`, in queue order.  Host only: no CUDA call.  Writes min(count,
 * max_pieces) entries of four ints to `pieces`: s0, s1, h0, h1, meaning
 * slices [s0, s1) whole (h0 = 0, h1 = G) or query heads [h0, h1) of slice s0
 * (s1 = s0 + 1), a slice being one (batch, key/value head) pair in batch-major
 * order.  `pieces` may be NULL when max_pieces is 0.  Returns the count, or
 * -TESSERA_ERR_INVALID_ARG for B, Hq, Hkv < 1, Hq % Hkv != 0, chunks < 0,
 * max_pieces < 0, or a NULL `pieces` with max_pieces > 0.
 */
int tessera_attn_fwd_host_plan(int B, int Hq, int Hkv, int chunks, int *pieces,
                               int max_pieces);

/*
 * One decoding step over a block-paged key/value cache.  The pages list a
 * fused paged-attention decode kernel as not yet built (hysenlabs.com Tessera
 * review, "The kernel set and its torch fallback"; sourcepulse.org Tessera
 * page, "Limitations & Caveats") beside the engine's block-paged KV cache
 * with a ref-counted allocator (Tessera README, "What's in it" / "Serving";
 * hysenlabs.com review, "Serving: block-paged KV, batch recomposition,
 * speculation").  They give no formula; the plain reading adopted here is the
 * forward's attention for one new query row per sequence over all of its
 * cached tokens, which are found through the block table:
 *
 *   n = seq_lens[b]; token j < n sits in block block_table[b][j / bs], row j % bs
 *   s_j = scale * dot(q[b,h,:], k_cache[blk, g, j % bs, :]),  g = floor(h / G)
 *   o[b,h,:] = sum_j softmax_j(s) * v_cache[blk, g, j % bs, :]
 *   lse[b,h] = ln sum_j exp(s_j)
 *
 * A sequence with n = 0 gets o = 0 and lse = -infinity.
 *
 * q            bf16 [B, Hq, d] device, read only (one query row per sequence)
 * k_cache,     bf16 [num_blocks, Hkv, block_size, d] device, read only; a block
 *   v_cache    holds block_size consecutive tokens of one sequence for every
 *              key/value head
 * block_table  int32 [B, max_blocks] device, read only; entries past a
 *              sequence's last block are not read
 * seq_lens     int32 [B] device, read only; each in 0 .. max_seq_len
 * o            bf16 [B, Hq, d] device, written
 * lse          fp32 [B, Hq] device, written; may be NULL
 * workspace    device memory of at least
 *              tessera_attn_decode_workspace_bytes(B, Hq, max_seq_len, d)
 *              bytes (may be NULL when that is 0), 16-byte aligned, owned by
 *              the caller; overwritten, nothing needs to be set before
 * B >= 0 (0 launches nothing); Hq, Hkv >= 1 with Hq % Hkv == 0;
 * d            64 or 128, block_size a power of two >= 8, else
 *              TESSERA_ERR_UNSUPPORTED
 * max_blocks, num_blocks >= 1; num_blocks * Hkv * block_size < 2^31
 * max_seq_len  host-side bound on seq_lens, 0 .. max_blocks * block_size;
 *              it sizes the launch and the workspace
 * scale        positive finite multiplier of q.k
 *
 * Checks before any CUDA call: sizes as above; q, caches, o, lse and the
 * workspace 16-byte aligned, the table and lengths 4-byte aligned
 * (TESSERA_ERR_MISALIGNED); no output (o, lse, workspace) overlapping an
 * input or another output (TESSERA_ERR_INVALID_ARG).  Device-resident values
 * are checked by the kernel: a length above max_seq_len (or negative) makes
 * that sequence empty, a block id outside 0 .. num_blocks-1 among the blocks
 * a sequence needs drops the 128-token part of the sequence holding it; both
 * record TESSERA_DEVICE_ERR_DECODE_INPUT for tessera_attn_device_error(), and
 * no memory outside the buffers above is read.  Queues up to two kernels on
 * `stream` (tessera_attn_last_launch_count() reports them) and does not
 * synchronise.
 */
#define TESSERA_DEVICE_ERR_DECODE_INPUT 20
size_t tessera_attn_decode_workspace_bytes(int B, int Hq, int max_seq_len, int d);
int tessera_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens, void *o,
                        float *lse, void *workspace, size_t workspace_bytes, int B, int Hq,
                        int Hkv, int d, int block_size, int max_blocks, int num_blocks,
                        int max_seq_len, float scale, tessera_stream_t stream);

/*
 * The attention block's prologue: the steps before attention in the pages'
 * decoder ("RMSNorm, RoPE, grouped-query attention and SwiGLU", Tessera
 * README, "What's in it" / "Training side"; its kernels include a fused
 * RMSNorm, README "What's in it" / "Kernels" and hysenlabs.com review, "The
 * kernel set and its torch fallback").  The pages give no formula; the plain
 * readings adopted here:
 *
 *   RMSNorm:  y[r,c] = x[r,c] / sqrt(mean_c x[r,c]^2 + eps) * w[c]
 *   RoPE of a head vector at position p, element i paired with i + d/2:
 *     theta_i = base^(-2i/d), a = p * theta_i
 *     y[i] = x[i] cos a - x[i+d/2] sin a,  y[i+d/2] = x[i] sin a + x[i+d/2] cos a
 *
 * Between the two runs the Q/K/V projection, a plain GEMM that is not part of
 * this library.  Both calls are asynchronous on `stream`, launch one kernel
 * (tessera_attn_last_launch_count() = 1, 0 when there is nothing to do),
 * allocate nothing, and check their arguments before any CUDA call.
 *
 * tessera_rmsnorm
 *   x    bf16 [rows, dim] device, read only
 *   w    bf16 [dim] device, read only
 *   y    bf16 [rows, dim] device, written (rounded to nearest even); may be x
 *        itself (in place), must not otherwise overlap x or w
 *   rows >= 0 (0 launches nothing); dim a multiple of 8 up to 8192, else
 *   TESSERA_ERR_UNSUPPORTED; eps >= 0 and finite.  Pointers 16-byte aligned.
 *   Sums of squares in fp32.
 */
int tessera_rmsnorm(const void *x, const void *w, void *y, int rows, int dim, float eps,
                    tessera_stream_t stream);

/*
 * tessera_rope_qkv: rotary embedding of the projected queries and keys, and
 * the split into the layout tessera_attn_fwd reads.
 *   qkv        bf16 [B, T, (Hq + 2*Hkv) * d] device, read only: per token the
 *              Hq query heads, then the Hkv key heads, then the Hkv value
 *              heads (the projection's output, token-major)
 *   positions  int32 [B, T] device, each token's position; NULL means p = t
 *   q          bf16 [B, Hq, T, d] device, written: rotated query heads
 *   k, v       bf16 [B, Hkv, T, d] device, written: rotated key heads, and the
 *              value heads copied
 *   B, T >= 0 (either 0 launches nothing); Hq, Hkv >= 1, Hq % Hkv == 0;
 *   d 64 or 128, else TESSERA_ERR_UNSUPPORTED; base > 0 and finite (10000 is
 *   the usual choice).  Pointers 16-byte aligned (positions 4-byte); q, k, v
 *   must not overlap qkv, positions or each other.  Angles are computed in
 *   fp64, the rotation in fp32.
 */
int tessera_rope_qkv(const void *qkv, const int32_t *positions, void *q, void *k, void *v,
                     int B, int T, int Hq, int Hkv, int d, float base,
                     tessera_stream_t stream);

/*
 * Reads and clears the device-side error word of the current device.  This
 * synchronises the device.  *code receives 0 when no kernel reported a
 * problem since the last call, else a nonzero code naming the wait that gave
 * up.  Returns TESSERA_OK, or TESSERA_ERR_CUDA if the read failed.
 */
int tessera_attn_device_error(int *code);

/*
 * Diagnostic of the bounded-wait machinery: queues on `stream` one warp that
 * waits, with the same bounded wait the attention kernel uses, on a barrier
 * that nothing completes.  The wait gives up after limit_us microseconds
 * (1 .. 10,000,000, else TESSERA_ERR_INVALID_ARG) and records code
 * TESSERA_DEVICE_ERR_SELFTEST in the device error word, which
 * tessera_attn_device_error() then returns.  Nothing faults or hangs and the
 * CUDA context stays usable.  Returns TESSERA_OK once queued.
 */
#define TESSERA_DEVICE_ERR_SELFTEST 9
int tessera_attn_selftest_timeout(unsigned int limit_us, tessera_stream_t stream);

/* A static string naming a tessera_status value. */
const char *tessera_status_str(int status);

/*
 * Kernel launches the last successful tessera_attn_fwd or
 * tessera_attn_fwd_varlen (0 or 1),
 * tessera_attn_fwd_host (one per chunk), tessera_attn_bwd (3),
 * tessera_attn_decode (1 or 2), tessera_rmsnorm or tessera_rope_qkv (1) call
 * on this thread queued.  Lets a caller
 * count the library's own launches.
 */
int tessera_attn_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TESSERA_ATTN_H */
