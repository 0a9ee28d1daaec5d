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
// byte, so it is bound by HBM bandwidth and runs on the FP32 pipes (packed
// f32x2 FMAs).  An item is one sequence and key/value head, for GT of its G
// query heads; its tokens form ceil(n / 128) chunks.
//   1. paged_decode_partial_kernel, persistent (one CTA per SM).  The chunks
//      of all items, item after item, form one stream; CTA k takes the k-th
//      of gridDim.x equal contiguous shares of it, so every SM moves the same
//      number of chunks whatever the lengths.  A producer warp finds its
//      share from the lengths and fills a ring of NS shared-memory stages by
//      TMA: a chunk's K and V pages (boxes of 64 columns x R rows, R =
//      min(bs, 128), 128-byte swizzle, evict-first in L2), plus the q rows at
//      the first chunk of an item.  Eight consumer warps run an online
//      softmax over the consecutive chunks of an item (a segment): per chunk,
//      scores (warp = column slice, lane = tokens, q in registers, swizzled K
//      rows read without bank conflicts), per head the running max m and sum
//      l with p = 2^(s - m), and p.V accumulated in registers (warp = column
//      slice, lanes = token slices x 4-column groups).  At a segment's end the
//      unnormalised o, m and l go to partial slot (item, k - first CTA of the
//      item); the CTA that ends an item records its slot count.
//   2. paged_decode_merge_kernel: a CTA per (b, h) combines the slots:
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

constexpr int kDecodeChunk = 128;                  // tokens per chunk
constexpr int kDecodeConsumers = 256;              // 8 consumer warps
constexpr int kDecodeThreads = 288;                // + the producer warp
constexpr int kDecodeProducerWarp = 8;
constexpr int kDecodeMaxBoxes = kDecodeChunk / 8;  // boxes per chunk at the smallest block size

// flags of a ring stage
constexpr int kStageBad = 1;        // a page of the chunk is not in the cache: skip it
constexpr int kStageSegFirst = 2;   // first chunk of this CTA's segment of the item (q copied)
constexpr int kStageSegLast = 4;    // last chunk of the segment: write the partial
constexpr int kStageItemLast = 8;   // last chunk of the item: record the slot count

template <int D, int GT>
struct DecodeCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static_assert(GT == 1 || GT == 2 || GT == 4 || GT == 8, "1, 2, 4 or 8 heads per item");
  static constexpr int CH = kDecodeChunk;
  static constexpr int NH = D / 64;      // 64-column halves (one TMA box width each)
  static constexpr int HALF = CH * 128;  // bytes of one half-tile [CH rows][64 cols]
  static constexpr int KV_BYTES = 2 * NH * HALF;  // K half-tiles, then V half-tiles
  static constexpr int Q_BYTES = GT * D * 2;      // the item's q rows (bf16)
  static constexpr int STAGE = (KV_BYTES + Q_BYTES + 1023) / 1024 * 1024;
  static constexpr int CPW = D / 8;               // columns per consumer warp
  // ring stages: 3 (d = 128) or 6 (d = 64), fewer where the scratch of 8 query
  // heads leaves no room
  static constexpr int NS_MAX = D == 128 ? 3 : 6;
  static constexpr int FIXED = GT * D * 4 + 8 * GT * CH * 4 + CH * GT * 4 + 32 + 48 * NS_MAX;
  static constexpr int NS_FIT = (232448 - 1024 - FIXED) / STAGE;
  static constexpr int NS = NS_FIT < NS_MAX ? NS_FIT : NS_MAX;
  static_assert(NS >= 2, "at least double buffering");
  static constexpr int SQ_OFF = NS * STAGE;               // float [GT][D]
  static constexpr int SP_OFF = SQ_OFF + GT * D * 4;      // float [8][GT][CH] partial scores
  static constexpr int P_OFF = SP_OFF + 8 * GT * CH * 4;  // float [CH][GT]
  static constexpr int AL_OFF = P_OFF + CH * GT * 4;      // float alpha[GT]
  static constexpr int META_OFF = AL_OFF + 32;            // int [NS][8]
  static constexpr int BAR_OFF = META_OFF + 32 * NS;      // full[NS], empty[NS]
  static constexpr int BYTES = BAR_OFF + 16 * NS;
  static constexpr int SMEM = BYTES + 1024;  // slack for the 1024-byte alignment
  static_assert(SMEM <= 232448, "fits the 227 KB a CTA may use");
};

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
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && ptx::globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Byte offset, in a [rows][64 cols] bf16 half-tile written by TMA with the
// 128-byte swizzle (1024-byte aligned), of the 16-byte chunk c of row r.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// bf16 pair (low half = lower column) -> fp32 pair
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
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
};

// Producer warp: this CTA's share [lo, hi) of the chunk stream, one ring
// stage per chunk, block ids of the next chunk read while the current one is
// issued.  Ends with a sentinel stage (b = -1).
template <int D, int GT>
__device__ __forceinline__ void decode_produce(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                               const DecodeParams& p, uint8_t* sm, int* meta,
                                               uint64_t* full, uint64_t* empty, int lane) {
  using C = DecodeCfg<D, GT>;
  const int R = p.rows_per_box;
  const long long HZ = static_cast<long long>(p.Hkv) * p.zgroups;
  // total chunks, then this CTA's share
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
    // the sequence holding stream position lo
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
        break;
      }
      pre = __shfl_sync(0xffffffffu, incl, 31);
    }
    const uint64_t pol = ptx::policy_evict_first();
    // block id of box `lane` of the chunk at `cu` (0 when the lane has none)
    auto load_ids = [&](const DecodeCursor& cu, int& blk, int& npg) {
      const int nt = min(C::CH, cu.n - cu.c * C::CH);
      npg = (nt + R - 1) / R;
      blk = 0;
      if (lane < npg)
        blk = p.block_table[static_cast<long long>(cu.b) * p.max_blocks +
                            (cu.c * C::CH + lane * R) / p.bs];
    };
    int blk, npg;
    load_ids(cur, blk, npg);
    for (long long pos = lo; pos < hi; ++pos) {
      // the next chunk's coordinates and block ids, read while this one is issued
      DecodeCursor nxt = cur;
      int nblk = 0, nnpg = 0;
      if (pos + 1 < hi) {
        if (++nxt.c == nxt.nchunks) {
          nxt.c = 0;
          nxt.item0 += nxt.nchunks;
          if (++nxt.gz == HZ) {  // next sequence with tokens
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
      const uint32_t s = produced % C::NS;
      bool ok = true;
      if (lane == 0) {
        if (bad) decode_error(p, kErrDecodeInput);
        ok = decode_wait(&empty[s], ((produced / C::NS) & 1) ^ 1u);
        if (!ok) decode_error(p, kErrDecodeWait);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        alive = false;
        break;
      }
      const int nt = min(C::CH, cur.n - cur.c * C::CH);
      const int g = cur.gz / p.zgroups, z = cur.gz % p.zgroups;
      if (lane == 0) {
        int* m = meta + 8 * s;
        m[0] = cur.b;
        m[1] = cur.gz;
        m[2] = cur.c;
        m[3] = nt;
        m[4] = flags;
        // partial slot: this CTA's index among the CTAs that share the item
        m[5] = static_cast<int>(blockIdx.x - cur.item0 / per);
        const uint32_t qb = seg_first && !bad ? C::Q_BYTES : 0;
        if (bad)
          ptx::mbar_arrive(&full[s]);
        else
          ptx::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(npg * R * D * 4) + qb);
        if (qb) {
          const long long head0 = static_cast<long long>(cur.b) * p.Hq + g * p.G + z * GT;
          ptx::bulk_load(sm + s * C::STAGE + C::KV_BYTES, p.q + head0 * D, C::Q_BYTES,
                         &full[s]);
        }
      }
      __syncwarp();
      if (!bad && lane < npg) {
        uint8_t* st = sm + s * C::STAGE;
        const int tok = cur.c * C::CH + lane * R;
        const int row = (blk * p.Hkv + g) * p.bs + tok % p.bs;
#pragma unroll
        for (int h = 0; h < C::NH; ++h)
          ptx::tma_load_2d_hint(st + h * C::HALF + lane * R * 128, tm_k, &full[s], 64 * h, row,
                                pol);
#pragma unroll
        for (int h = 0; h < C::NH; ++h)
          ptx::tma_load_2d_hint(st + (C::NH + h) * C::HALF + lane * R * 128, tm_v, &full[s],
                                64 * h, row, pol);
      }
      ++produced;
      cur = nxt;
      blk = nblk;
      npg = nnpg;
    }
  }
  if (alive && lane == 0) {
    const uint32_t s = produced % C::NS;
    if (decode_wait(&empty[s], ((produced / C::NS) & 1) ^ 1u)) {
      meta[8 * s] = -1;
      ptx::mbar_arrive(&full[s]);
    } else {
      decode_error(p, kErrDecodeWait);
    }
  }
}

// The eight consumer warps: the stages in the producer's order.
template <int D, int GT>
__device__ __forceinline__ void decode_consume(const DecodeParams& p, uint8_t* sm, int* meta,
                                               uint64_t* full, uint64_t* empty, int tid) {
  using C = DecodeCfg<D, GT>;
  constexpr int CPW = C::CPW;   // columns per warp (16 or 8)
  constexpr int CGW = CPW / 4;  // 4-column groups per warp (phase 3)
  constexpr int SL = 32 / CGW;  // token slices (phase 3)
  float* sq = reinterpret_cast<float*>(sm + C::SQ_OFF);
  float* sp = reinterpret_cast<float*>(sm + C::SP_OFF);
  float* spp = reinterpret_cast<float*>(sm + C::P_OFF);
  float* salpha = reinterpret_cast<float*>(sm + C::AL_OFF);
  const int warp = tid >> 5, lane = tid & 31;
  // running max / sum of head `warp` (warps < GT), the same in every lane
  float m_run = -INFINITY, l_run = 0.f;
  // p.V accumulators of columns col3 .. col3+3: one head (GT = 1) as column
  // pairs acc[0][0..1]; else head pairs acc3[hp][e] = (head 2hp, 2hp+1) of
  // column col3 + e
  float2 acc[1][2];
  float2 acc3[GT / 2 > 0 ? GT / 2 : 1][4];
  acc[0][0] = acc[0][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int hp = 0; hp < (GT / 2 > 0 ? GT / 2 : 1); ++hp)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc3[hp][e] = make_float2(0.f, 0.f);
  const int cg = lane % CGW, slice = lane / CGW;
  const int col3 = warp * CPW + 4 * cg;  // phase 3 columns col3 .. col3+3
  for (uint32_t k = 0;; ++k) {
    const uint32_t s = k % C::NS;
    bool ok = decode_wait(&full[s], (k / C::NS) & 1);
    ok = ptx::bar_red_and(1, kDecodeConsumers, ok);
    if (!ok) {
      if (tid == 0) decode_error(p, kErrDecodeWait);
      return;
    }
    const int* m = meta + 8 * s;
    const int b = m[0];
    if (b < 0) return;  // the producer's sentinel
    const int gz = m[1], nt = m[3], flags = m[4], slot = m[5];
    const int g = gz / p.zgroups, z = gz % p.zgroups;
    const long long head0 = static_cast<long long>(b) * p.Hq + g * p.G + z * GT;
    const uint8_t* st = sm + s * C::STAGE;
    if (!(flags & kStageBad)) {
      if (flags & kStageSegFirst) {
        const __nv_bfloat16* sqb = reinterpret_cast<const __nv_bfloat16*>(st + C::KV_BYTES);
        for (int i = tid; i < GT * D; i += kDecodeConsumers)
          sq[i] = __bfloat162float(sqb[i]) * p.scale_log2;
        ptx::bar_sync_named(1, kDecodeConsumers);
      }
      // 1. partial scores over this warp's CPW columns, tokens lane + 32 r;
      // heads in groups of up to 4 (q of a group in registers).  Row t's
      // swizzle phase is t & 7 = lane & 7, so a lane's K offsets are fixed.
      {
        constexpr int HG = GT < 4 ? GT : 4;
        constexpr int KC = CPW / 8;  // 16-byte chunks per row slice
        uint32_t koff[KC];
#pragma unroll
        for (int j = 0; j < KC; ++j) {
          const int gc = warp * KC + j;
          koff[j] = static_cast<uint32_t>((gc >> 3) * C::HALF + lane * 128 +
                                          (((gc & 7) ^ (lane & 7)) << 4));
        }
        const bool full_chunk = nt == C::CH;
#pragma unroll
        for (int h0 = 0; h0 < GT; h0 += HG) {
          float2 qp[HG][CPW / 2];
#pragma unroll
          for (int gh = 0; gh < HG; ++gh)
#pragma unroll
            for (int j = 0; j < CPW / 4; ++j) {
              const float4 x =
                  *reinterpret_cast<const float4*>(sq + (h0 + gh) * D + warp * CPW + 4 * j);
              qp[gh][2 * j] = make_float2(x.x, x.y);
              qp[gh][2 * j + 1] = make_float2(x.z, x.w);
            }
          auto token = [&](int r) {
            float2 kp[CPW / 2];
#pragma unroll
            for (int j = 0; j < KC; ++j) {
              const uint4 u = *reinterpret_cast<const uint4*>(st + koff[j] + r * 32 * 128);
              kp[4 * j] = bf16x2_to_f2(u.x);
              kp[4 * j + 1] = bf16x2_to_f2(u.y);
              kp[4 * j + 2] = bf16x2_to_f2(u.z);
              kp[4 * j + 3] = bf16x2_to_f2(u.w);
            }
#pragma unroll
            for (int gh = 0; gh < HG; ++gh) {
              float2 acc2 = __fmul2_rn(kp[0], qp[gh][0]);
#pragma unroll
              for (int j = 1; j < CPW / 2; ++j) acc2 = __ffma2_rn(kp[j], qp[gh][j], acc2);
              sp[(warp * GT + h0 + gh) * C::CH + lane + 32 * r] = acc2.x + acc2.y;
            }
          };
          if (full_chunk) {
#pragma unroll
            for (int r = 0; r < C::CH / 32; ++r) token(r);
          } else {
#pragma unroll
            for (int r = 0; r < C::CH / 32; ++r)
              if (lane + 32 * r < nt) token(r);
          }
        }
      }
      ptx::bar_sync_named(1, kDecodeConsumers);

      // 2. per head (warp gh): scores, running max, p = 2^(s - m), running sum
      if (warp < GT) {
        const int gh = warp;
        float sv[C::CH / 32];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < C::CH / 32; ++j) {
          const int t = lane + 32 * j;
          float x = -INFINITY;
          if (t < nt) {
            x = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) x += sp[(w * GT + gh) * C::CH + t];
          }
          sv[j] = x;
          mx = fmaxf(mx, x);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = ptx::ex2(m_run - m_new);  // 0 at a segment's first chunk
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < C::CH / 32; ++j) {
          const float e = ptx::ex2(sv[j] - m_new);  // masked tokens: 2^-inf = 0
          spp[(lane + 32 * j) * GT + gh] = e;
          sum += e;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        l_run = fmaf(l_run, alpha, sum);
        m_run = m_new;
        if (lane == 0) salpha[gh] = alpha;
      }
      ptx::bar_sync_named(1, kDecodeConsumers);

      // 3. acc = alpha * acc + sum_i p[i] v_i over this lane's tokens
      // i = slice + SL j, whose swizzle phase i & 7 = slice & 7 is fixed
      {
        const int gc = col3 >> 3;
        const uint8_t* vl = st + (C::NH + (gc >> 3)) * C::HALF + ((col3 & 7) << 1) +
                            slice * 128 + (((gc & 7) ^ (slice & 7)) << 4);
        const float* pl = spp + slice * GT;
        if constexpr (GT == 1) {
          const float2 a2 = make_float2(salpha[0], salpha[0]);
          acc[0][0] = __fmul2_rn(acc[0][0], a2);
          acc[0][1] = __fmul2_rn(acc[0][1], a2);
        } else {
#pragma unroll
          for (int hp = 0; hp < GT / 2; ++hp) {
            const float2 a2 = *reinterpret_cast<const float2*>(salpha + 2 * hp);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc3[hp][e] = __fmul2_rn(acc3[hp][e], a2);
          }
        }
        auto token = [&](int j) {
          const uint2 u = *reinterpret_cast<const uint2*>(vl + j * SL * 128);
          const float* pi = pl + j * SL * GT;
          if constexpr (GT == 1) {
            // column pairs, p duplicated
            const float2 pp = make_float2(pi[0], pi[0]);
            acc[0][0] = __ffma2_rn(bf16x2_to_f2(u.x), pp, acc[0][0]);
            acc[0][1] = __ffma2_rn(bf16x2_to_f2(u.y), pp, acc[0][1]);
          } else {
            // head pairs: p of two heads is one load, v duplicated
            const float v[4] = {__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u)};
#pragma unroll
            for (int hp = 0; hp < GT / 2; ++hp) {
              const float2 pp = *reinterpret_cast<const float2*>(pi + 2 * hp);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                acc3[hp][e] = __ffma2_rn(make_float2(v[e], v[e]), pp, acc3[hp][e]);
            }
          }
        };
        if (nt == C::CH) {
#pragma unroll
          for (int j = 0; j < C::CH / SL; ++j) token(j);
        } else {
#pragma unroll 4
          for (int j = 0; slice + j * SL < nt; ++j) token(j);
        }
      }
    }
    // every read of this stage is done: hand it back to the producer
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[s]);

    if (flags & kStageSegLast) {
      const long long base = head0 * p.nslot + slot;  // slot of head gh: + gh * nslot
      float o4[GT][4];
      if constexpr (GT == 1) {
        o4[0][0] = acc[0][0].x;
        o4[0][1] = acc[0][0].y;
        o4[0][2] = acc[0][1].x;
        o4[0][3] = acc[0][1].y;
        acc[0][0] = acc[0][1] = make_float2(0.f, 0.f);
      } else {
#pragma unroll
        for (int hp = 0; hp < GT / 2; ++hp)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o4[2 * hp][e] = acc3[hp][e].x;
            o4[2 * hp + 1][e] = acc3[hp][e].y;
            acc3[hp][e] = make_float2(0.f, 0.f);
          }
      }
#pragma unroll
      for (int msk = CGW; msk < 32; msk <<= 1)
#pragma unroll
        for (int gh = 0; gh < GT; ++gh)
#pragma unroll
          for (int e = 0; e < 4; ++e) o4[gh][e] += __shfl_xor_sync(0xffffffffu, o4[gh][e], msk);
      if (slice == 0) {
#pragma unroll
        for (int gh = 0; gh < GT; ++gh)
          *reinterpret_cast<float4*>(p.part_o + (base + gh * p.nslot) * D + col3) =
              make_float4(o4[gh][0], o4[gh][1], o4[gh][2], o4[gh][3]);
      }
      if (warp < GT) {
        if (lane == 0) {
          float* ml = p.part_ml + (base + warp * p.nslot) * 2;
          ml[0] = m_run;
          ml[1] = l_run;
        }
        m_run = -INFINITY;
        l_run = 0.f;
      }
      if ((flags & kStageItemLast) && tid == 0)
        p.slots[static_cast<long long>(b) * p.Hkv * p.zgroups + gz] = slot + 1;
    }
  }
}

template <int D, int GT>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    paged_decode_partial_kernel(const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeCfg<D, GT>;
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  int* meta = reinterpret_cast<int*>(sm + C::META_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* empty = full + C::NS;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kDecodeConsumers / 32);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if ((tid >> 5) == kDecodeProducerWarp)
    decode_produce<D, GT>(&tm_k, &tm_v, p, sm, meta, full, empty, tid & 31);
  else
    decode_consume<D, GT>(p, sm, meta, full, empty, tid);
}

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
