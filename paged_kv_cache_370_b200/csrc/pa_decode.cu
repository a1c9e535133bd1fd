// pa_decode.cu -- paged decode attention for sm_100a.
//
// What it computes (pages: "大语言模型推理内存管理算法 paged attention",
// sections 5-6; "08. PagedAttention：把 KV Cache 分页管理", sections
// "为什么叫 PagedAttention" and "它没有解决什么"; "PagedAttention 核心思想解析",
// section 2.2): for each sequence b and query head h,
//     out[b,h] = softmax(scale * q[b,h] . K_b^T) V_b
// over the sequence's whole history, where token t's K/V row lives in
// physical block block_tables[b][t / block_size] at offset t % block_size.
// Partial results over parts of the history are merged by log-sum-exp.
//
// Design (B200):
//  * One CTA per (split-context partition, kv head, sequence). The q heads of
//    the GQA group that share the kv head are processed together, so every
//    K/V byte is read from HBM once per step.
//  * A producer warp streams the partition's K and V tiles of TILE tokens into
//    a ring of NSTAGES shared-memory stages with 1-D TMA bulk copies
//    (cp.async.bulk ... mbarrier::complete_tx): one copy per (block, kv head)
//    piece, which is a contiguous run of rows in the pool, so each block is
//    read as whole coalesced rows. Full/empty mbarriers order the ring.
//  * Four consumer warps split each tile by tokens. A token's head_dim
//    elements are spread over LPT = head_dim / 8 lanes (16 bytes each); each
//    lane keeps its q chunk for all G heads in registers, forms G partial dot
//    products and a reduce-scatter over the LPT lanes leaves every lane one
//    head's full score. Scores are kept in the log2 domain.
//  * Online softmax per token group: tile max, one rescale of the running
//    (max, sum, weighted V) state per tile, exp2 of the scores; the G heads'
//    weights are shared through a small shared-memory slot.
//  * The CTA's token groups are merged in a fixed order (deterministic; the
//    result depends only on logical token order, never on physical ids or
//    the block size). A single-partition sequence writes its output
//    directly; otherwise the partition writes (max, sum, weighted V) to the
//    workspace and pa_decode_merge_kernel combines the partitions.
//  * Every wait is bounded in wall-clock time; a block id or length out of
//    range is skipped and reported in the device error word, never accessed.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace {

__device__ int g_decode_error;

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 4;
constexpr int kTileBytes = 8192;                 // bytes of K (and of V) per stage
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
// how long the decode consumers wait for the producer's word on the piece it may
// fetch before their final merge (it comes one counter read after the producer's
// last copies are issued); then they go ahead without it
constexpr unsigned long long kPreWaitNs = 20000ull;  // 20 us

// Wait for phase `parity` of `bar` to complete, at most limit_ns; also give up
// when another thread of the CTA has raised *abort. Returns false on give-up
// (and then raises *abort and the device error bit).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort = 1;
      atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// The same wait without the early exit on *abort: for barriers whose arrivals
// do not depend on any copy landing (they always come), so that a give-up
// elsewhere in the CTA cannot let one warp run ahead of another.
__device__ __forceinline__ bool mbar_wait_sure(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// ------------------------------------------------------------------- reduce-scatter over lanes
// N values per lane, over the lanes of one token group (offsets O, O/2, ...):
// each halving level keeps half of the values, adding the partner's copy, so
// after log2(N) levels a lane holds one value summed over 2^log2(N) lanes.
template <int N, int O>
struct HalvingSum {
  static __device__ __forceinline__ void run(float *v, int lane) {
    const bool upper = (lane & O) != 0;
#pragma unroll
    for (int j = 0; j < N / 2; ++j) {
      const float send = upper ? v[j] : v[j + N / 2];
      const float keep = upper ? v[j + N / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    HalvingSum<N / 2, O / 2>::run(v, lane);
  }
};
template <int O>
struct HalvingSum<1, O> {
  static __device__ __forceinline__ void run(float *, int) {}
};

// Full sum of value v over lanes differing in the bits below O*2 (butterfly).
template <int O>
__device__ __forceinline__ float butterfly_sum(float v) {
#pragma unroll
  for (int o = O; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// --------------------------------------------------------------------------------- parameters
struct DecodeParams {
  void *out;
  const void *q;
  const void *k_cache;
  const void *v_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *ws_acc;  // [B][Hq][max_parts][D]
  float *ws_ml;   // [B][Hq][max_parts][2] = (max in log2 units, sum)
  int max_blocks_per_seq;
  int max_context_len;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int partition_tokens;
  int max_parts;
  int table_slice;  // shared-memory entries reserved for a partition's block ids
  float scale_log2;  // scale * log2(e)
  // even-split (persistent) kernel only
  int num_seqs;
  int grid_ctas;       // CTAs sharing the tiles
  int *ws_counters;    // [grid_ctas] pieces finished per split segment; zero between calls
  float *ws_pieces;    // [2 * grid_ctas][G][D + 4] partial (acc[D], max, sum, pad) per piece
  // fused KV write (pa_decode_append): the new token of sequence b is position
  // context_lens[b] - 1, with rows k_new[b], v_new[b] and slot new_slots[b]
  const void *k_new;
  const void *v_new;
  const int64_t *new_slots;  // nullptr: no fused write
  void *k_cache_w;
  void *v_cache_w;
  // sliding window: a sequence of length len attends to positions
  // [len - window, len) (0: every position). The partition kernel applies it
  // directly; the even-split kernel (its kWindow instantiation) sees each
  // sequence from the block holding its first attended position on (seq_view)
  int window;
  // even-split kernel launched as a programmatic dependent of the preceding kernel
  int early_start;
  // limit of the consumers' waits for a stage's data (normally kWaitLimitNs)
  unsigned long long wait_ns;
  // test mode of the bounded waits: the producers issue no copy and arrive on no
  // data barrier, so every data wait runs out (pa_debug_wait_test)
  int starve;
};

// First position attended by a sequence of length len under a window of w
// positions (w <= 0: no window).
__device__ __forceinline__ int window_lo(int len, int w) { return w > 0 && len > w ? len - w : 0; }

template <int D>
struct Shape {
  static constexpr int kLpt = D / 8;                         // lanes per token (16 B each)
  static constexpr int kGroupsPerWarp = 32 / kLpt;           // token groups per warp
  static constexpr int kGroups = kConsumerWarps * kGroupsPerWarp;
  static constexpr int kTile = kTileBytes / (D * 2);         // tokens per stage
  static constexpr int kTokPerGroup = kTile / kGroups;       // tokens per group per tile
  static_assert(kTokPerGroup >= 1 && kTile % kGroups == 0, "tile split");
};

template <typename T, int D, int G>
struct Smem {
  using S = Shape<D>;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile then V tile
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kRedBytes = S::kGroups * G * D * 4;  // final cross-group merge
  static_assert(kRedBytes <= kRingBytes, "merge buffer must fit in the ring");
  static constexpr int kPbufFloats = S::kGroups * (S::kTokPerGroup + 1) * G;
  static constexpr int kMlFloats = S::kGroups * G * 2;
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kPbufOffset = kBarOffset + 2 * kStages * 8;
  static constexpr int kMlOffset = kPbufOffset + kPbufFloats * 4;
  static constexpr int kFlagOffset = kMlOffset + kMlFloats * 4;
  static constexpr int kTableOffset = kFlagOffset + 16;
  static size_t bytes(int table_slice) { return kTableOffset + (size_t)table_slice * 4; }
};

// ------------------------------------------------------------------------------ main kernel
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 3)
    pa_decode_partition_kernel(const DecodeParams p) {
  using S = Shape<D>;
  using L = Smem<T, D, G>;
  constexpr int LPT = S::kLpt;
  constexpr int TILE = S::kTile;
  constexpr int TPG = S::kTokPerGroup;
  constexpr int NG = S::kGroups;
  constexpr int CH = 8;  // elements per lane chunk

  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *empty_bar = full_bar + kStages;
  float *pbuf = reinterpret_cast<float *>(smem + L::kPbufOffset);
  float *mlbuf = reinterpret_cast<float *>(smem + L::kMlOffset);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kFlagOffset);
  int32_t *table = reinterpret_cast<int32_t *>(smem + L::kTableOffset);

  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- the partition's token range
  int len = __ldg(p.context_lens + b);
  const int cap = p.max_blocks_per_seq * p.block_size;
  if (len < 0 || len > cap || len > p.max_context_len) {
    if (tid == 0 && part == 0 && kvh == 0) atomicOr(&g_decode_error, PA_DEVERR_CONTEXT_LEN);
    len = len < 0 ? 0 : min(min(len, cap), p.max_context_len);
  }
  // partitions cover [lo, len): blocks before a sliding window are never read
  const int lo = window_lo(len, p.window);
  const int nparts = len > lo ? (len - lo + p.partition_tokens - 1) / p.partition_tokens : 1;
  if (part >= nparts) return;
  const int t_begin = lo + part * p.partition_tokens;
  const int t_end = min(len, t_begin + p.partition_tokens);
  const int ntok = t_end - t_begin;  // may be 0 only for an empty sequence
  const int ntiles = (ntok + TILE - 1) / TILE;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the producer warp stages the partition's block ids
  const int blk_first = t_begin / p.block_size;
  const int nblk = ntok > 0 ? (t_end - 1) / p.block_size - blk_first + 1 : 0;
  if (warp == kConsumerWarps) {
    const int32_t *row = p.block_tables + (size_t)b * p.max_blocks_per_seq + blk_first;
    for (int i = lane; i < nblk; i += 32) table[i] = __ldg(row + i);
  }
  __syncthreads();

  const size_t head_stride = (size_t)p.block_size * D;      // elements per (block, head) tile
  const size_t block_stride = head_stride * p.num_kv_heads;  // elements per block

  if (warp == kConsumerWarps) {
    // =============================================================== producer
    if (lane == 0) {
      const T *kc = static_cast<const T *>(p.k_cache);
      const T *vc = static_cast<const T *>(p.v_cache);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages &&
            !mbar_wait_bounded(&empty_bar[s], ((i / kStages) & 1) ^ 1, abort_flag))
          break;
        const int t0 = t_begin + i * TILE;
        const int t1 = min(t0 + TILE, t_end);
        // validate the pieces first, so the expected byte count is exact
        uint32_t bytes = 0;
        for (int blk = t0 / p.block_size; blk <= (t1 - 1) / p.block_size; ++blk) {
          const int r0 = max(t0, blk * p.block_size), r1 = min(t1, (blk + 1) * p.block_size);
          const int phys = table[blk - blk_first];
          if (phys < 0 || phys >= p.num_blocks) {
            atomicOr(&g_decode_error, PA_DEVERR_BLOCK_ID);
            continue;
          }
          bytes += 2u * (uint32_t)(r1 - r0) * D * sizeof(T);
        }
        if (p.starve) {  // test mode: no copy, no arrival (the consumers' waits run out)
          issued = i + 1;
          continue;
        }
        mbar_expect_tx_arrive(&full_bar[s], bytes);
        unsigned char *stage = smem + s * L::kStageBytes;
        for (int blk = t0 / p.block_size; blk <= (t1 - 1) / p.block_size; ++blk) {
          const int r0 = max(t0, blk * p.block_size), r1 = min(t1, (blk + 1) * p.block_size);
          const int phys = table[blk - blk_first];
          if (phys < 0 || phys >= p.num_blocks) continue;
          const size_t src = (size_t)phys * block_stride + (size_t)kvh * head_stride +
                             (size_t)(r0 - blk * p.block_size) * D;
          const uint32_t nbytes = (uint32_t)(r1 - r0) * D * sizeof(T);
          const int row = r0 - t0;
          bulk_g2s(stage + row * D * sizeof(T), kc + src, nbytes, &full_bar[s]);
          bulk_g2s(stage + kTileBytes + row * D * sizeof(T), vc + src, nbytes, &full_bar[s]);
        }
        issued = i + 1;
      }
      // do not leave while copies may still land in this CTA's shared memory
      for (int i = max(0, issued - kStages); i < issued && !p.starve; ++i) {
        const int s = i % kStages;
        const unsigned long long t_start = global_ns();
        while (!mbar_try_wait(&full_bar[s], (i / kStages) & 1)) {
          if (global_ns() - t_start > kWaitLimitNs) {
            atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
            break;
          }
        }
      }
    }
    return;
  }

  // =================================================================== consumers
  const int grp = warp * S::kGroupsPerWarp + lane / LPT;  // token group in the CTA
  const int li = lane % LPT;                               // lane within the group
  const int c = li;                                        // this lane's 8-element chunk
  const int hq0 = kvh * G;                                 // first q head of the group

  // q chunk for the G heads, fp32
  float qf[G][CH];
  {
    const uint4 *qv = static_cast<const uint4 *>(p.q);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint4 r = __ldg(qv + (((size_t)b * p.num_q_heads + hq0 + h) * D) / CH + c);
      Elem<T>::to_f32(r, qf[h]);
    }
  }
  // head whose score this lane owns after the reduce-scatter
  int hh = 0;
  {
    int n = G, o = LPT / 2;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      if (n > 1) {
        if (li & o) hh += n / 2;
        n >>= 1;
        o >>= 1;
      }
    }
  }
  const bool writer = (li & (LPT / G - 1)) == 0;
  float *gp = pbuf + grp * (TPG + 1) * G;  // this group's weights slot

  float m_run = -INFINITY;  // running max of head hh (log2 units)
  float l_run = 0.f;        // running sum of head hh
  float acc[G][CH];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < CH; ++e) acc[h][e] = 0.f;

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    // every lane waits; the warp then leaves together or not at all, so the
    // warp-wide shuffles below always see all 32 lanes
    const bool landed = mbar_wait_bounded(&full_bar[s], (i / kStages) & 1, abort_flag, p.wait_ns);
    if (!__all_sync(0xffffffffu, landed)) break;
    const unsigned char *stage = smem + s * L::kStageBytes;
    const uint4 *Ks = reinterpret_cast<const uint4 *>(stage);
    const uint4 *Vs = reinterpret_cast<const uint4 *>(stage + kTileBytes);
    const int nvalid = min(TILE, t_end - (t_begin + i * TILE));
    const int tbase = grp * TPG;

    // scores of this group's tokens (head hh), log2 units; -inf when masked.
    // The shuffles run for every token slot in every lane (a slot past the
    // valid rows reads stale but in-bounds stage memory and is then masked
    // by a select), so no shuffle is ever issued by part of a warp.
    float sc[TPG];
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      const int t = tbase + j;
      float kf[CH];
      Elem<T>::to_f32(Ks[t * (D / CH) + c], kf);
      float part[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < CH; ++e) a = fmaf(qf[h][e], kf[e], a);
        part[h] = a;
      }
      HalvingSum<G, LPT / 2>::run(part, lane);
      const float sj = butterfly_sum<LPT / (2 * G)>(part[0]) * p.scale_log2;
      sc[j] = (t < nvalid) ? sj : -INFINITY;
    }
    float m_tile = sc[0];
#pragma unroll
    for (int j = 1; j < TPG; ++j) m_tile = fmaxf(m_tile, sc[j]);
    const float m_new = fmaxf(m_run, m_tile);
    const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
    float w[TPG];
    float wsum = 0.f;
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      w[j] = (sc[j] == -INFINITY) ? 0.f : exp2f(sc[j] - m_new);
      wsum += w[j];
    }
    l_run = l_run * alpha + wsum;
    m_run = m_new;

    // share the G heads' weights and rescale factors within the group
    float wa[TPG][G];
    float al[G];
    if constexpr (G == 1) {
      al[0] = alpha;
#pragma unroll
      for (int j = 0; j < TPG; ++j) wa[j][0] = w[j];
    } else {
      if (writer) {
#pragma unroll
        for (int j = 0; j < TPG; ++j) gp[j * G + hh] = w[j];
        gp[TPG * G + hh] = alpha;
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j <= TPG; ++j) {
        float *dst = (j < TPG) ? wa[j] : al;
        const float *src = gp + j * G;
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int h = 0; h < G; h += 4) {
            const float4 v4 = *reinterpret_cast<const float4 *>(src + h);
            dst[h] = v4.x;
            dst[h + 1] = v4.y;
            dst[h + 2] = v4.z;
            dst[h + 3] = v4.w;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) dst[h] = src[h];
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < CH; ++e) acc[h][e] *= al[h];
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      const int t = tbase + j;
      if (t < nvalid) {
        float vf[CH];
        Elem<T>::to_f32(Vs[t * (D / CH) + c], vf);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < CH; ++e) acc[h][e] = fmaf(wa[j][h], vf[e], acc[h][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }

  // ---- merge the token groups of the CTA (fixed order)
  if (writer) {
    mlbuf[(grp * G + hh) * 2] = m_run;
    mlbuf[(grp * G + hh) * 2 + 1] = l_run;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  float Mh[G], Lh[G], fac[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
    for (int gg = 0; gg < NG; ++gg) M = fmaxf(M, mlbuf[(gg * G + h) * 2]);
    float Ls = 0.f;
    for (int gg = 0; gg < NG; ++gg) {
      const float mg = mlbuf[(gg * G + h) * 2];
      if (mg != -INFINITY) Ls += exp2f(mg - M) * mlbuf[(gg * G + h) * 2 + 1];
    }
    Mh[h] = M;
    Lh[h] = Ls;
    const float mine = mlbuf[(grp * G + h) * 2];
    fac[h] = (mine == -INFINITY) ? 0.f : exp2f(mine - M);
  }
  float *red = reinterpret_cast<float *>(smem);  // [NG][G][D]; the ring is idle now
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float4 *dst = reinterpret_cast<float4 *>(red + ((size_t)grp * G + h) * D + c * CH);
    dst[0] = make_float4(acc[h][0] * fac[h], acc[h][1] * fac[h], acc[h][2] * fac[h],
                         acc[h][3] * fac[h]);
    dst[1] = make_float4(acc[h][4] * fac[h], acc[h][5] * fac[h], acc[h][6] * fac[h],
                         acc[h][7] * fac[h]);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

  const bool single = (nparts == 1);
  constexpr int kOutPerThread = 4;
  for (int e0 = tid * kOutPerThread; e0 < G * D; e0 += kConsumerWarps * 32 * kOutPerThread) {
    const int h = e0 / D, d = e0 % D;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int gg = 0; gg < NG; ++gg) {
      const float4 v = *reinterpret_cast<const float4 *>(red + ((size_t)gg * G + h) * D + d);
      sum.x += v.x;
      sum.y += v.y;
      sum.z += v.z;
      sum.w += v.w;
    }
    float Lsel = 0.f, Msel = 0.f;
#pragma unroll
    for (int hx = 0; hx < G; ++hx)
      if (hx == h) {
        Lsel = Lh[hx];
        Msel = Mh[hx];
      }
    const size_t hq = (size_t)b * p.num_q_heads + hq0 + h;
    if (single) {
      const float inv = Lsel > 0.f ? 1.f / Lsel : 0.f;
      T *out = static_cast<T *>(p.out);
      *reinterpret_cast<uint2 *>(out + hq * D + d) =
          Elem<T>::from_f32x4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
    } else {
      *reinterpret_cast<float4 *>(p.ws_acc + (hq * p.max_parts + part) * D + d) = sum;
      if (d == 0) {
        p.ws_ml[(hq * p.max_parts + part) * 2] = Msel;
        p.ws_ml[(hq * p.max_parts + part) * 2 + 1] = Lsel;
      }
    }
  }
}

// ===================================================================== tensor-core variant
// pa_decode_stream_kernel: paged decode on tensor cores with an even split of the
// whole batch over one persistent wave of CTAs.
//  * The work is the list of (sequence, kv head) segments, each cut into tiles of
//    64 tokens; W tiles in all. CTA c takes tiles [c*W/n, (c+1)*W/n): every CTA
//    streams the same number of tiles (+-1) through one continuous pipeline, so
//    neither uneven lengths nor per-partition ramp-up leave the HBM idle. The
//    split points depend only on token counts, never on block ids or sizes.
//  * A producer warp walks the CTA's tiles in order and stages each (block, kv
//    head) piece with 2-D TMA tensor copies (cp.async.bulk.tensor, 128-byte
//    swizzle, no multicast) into 1024-byte-aligned panels of 64 head_dim
//    columns x 64 tokens; at the start of a segment it also copies the GQA
//    group's q rows. Per-tile metadata travels with the stage.
//  * Each consumer warp owns 16 tokens of a tile and computes S^T = K_tile . Q^T
//    with mma.m16n8k16 (tokens are M, the GQA group padded to 8 is N, head_dim
//    is K). The score fragment, turned into weights P and transposed in
//    registers with movmatrix, is the B operand of O^T += V_tile^T . P (head_dim
//    is M): weights never touch shared memory.
//  * Weights are rounded to the input type for the product and the running sum
//    uses the same rounded values, so the result is an exact weighted average of
//    V with each weight perturbed by at most one rounding. The running output is
//    rescaled only when some head's max grew.
//  * When a CTA reaches the end of its piece of a segment, its warps merge in a
//    fixed order. A segment wholly inside the CTA is written out directly.
//    Otherwise the piece's (acc, max, sum) goes to the workspace and a counter
//    per split segment is incremented; the CTA that brings it to the number of
//    pieces merges them (in CTA order: deterministic) and resets the counter,
//    so the counters are zero again when the kernel ends. No CTA ever waits for
//    another.
// Requires a power-of-two block size >= 8 (every TMA box then starts on a
// 1024-byte boundary and blocks align with 64-token tiles).
// Pipeline depth of the even-split kernel (stages of 64 tokens of K and V).
#ifndef PA_STREAM_STAGES_D128
#define PA_STREAM_STAGES_D128 3
#endif
#ifndef PA_STREAM_STAGES_D64
#define PA_STREAM_STAGES_D64 4
#endif


namespace tc {

constexpr int kTile = 64;            // tokens per stage
constexpr int kWarps = 4;            // consumer warps, 16 tokens each
// two producer warps: warp kWarps stages K (plus per-tile metadata, q rows and
// the new token), warp kWarps + 1 stages V. Issuing tensor copies takes the
// issuing warp time in proportion to the bytes, so one issuer per CTA would cap
// the CTA below its share of HBM bandwidth.
constexpr int kThreads = (kWarps + 2) * 32;
constexpr int kPanelBytes = kTile * 128;  // 64 columns of 2 bytes x 64 rows
constexpr int kIdWindow = 8;             // tiles of block ids fetched ahead of their copies
constexpr int kScanLoads = 8;            // lengths per lane loaded at once when sizing the job

// Per-tile schedule handed from the producer warp to the consumers with the tile.
struct TileMeta {
  int b, kvh, j;      // sequence, kv head, tile index inside the (sequence, kv head) segment
  int seg_tiles;      // tiles of the segment
  int nvalid;         // valid tokens in this tile (0..64)
  int seg_first_x;    // global index of the segment's first tile
  int flags;          // 1: first tile of this CTA's piece, 2: last tile of it,
                      // 4: holds the sequence's new token (fused write)
  int nskip;          // leading rows before a sliding window (the segment's first tile)
  long long new_slot;  // slot of the new token (flags & 4)
};

template <int D, int G>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kStageBytes = 2 * kPanels * kPanelBytes;  // K panels then V panels
  static constexpr int kStages = D == 128 ? PA_STREAM_STAGES_D128 : PA_STREAM_STAGES_D64;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kQBytes = G * D * 2;  // the q rows of one GQA group
  static constexpr int kQOffset = kRingBytes;
  static constexpr int kNewBytes = 2 * D * 2;  // the new token's K and V rows
  static constexpr int kNewOffset = kQOffset + kStages * kQBytes;
  static constexpr int kRedOffset = kNewOffset + kStages * kNewBytes;
  static constexpr int kRedBytes = kWarps * G * D * 4;
  static constexpr int kMetaOffset = kRedOffset + kRedBytes;
  static constexpr int kBarOffset = kMetaOffset + kStages * (int)sizeof(TileMeta);
  static constexpr int kMlOffset = kBarOffset + 2 * kStages * 8;  // full, empty barriers
  static constexpr int kIdsOffset = kMlOffset + kWarps * 8 * 2 * 4;
  // CTAs per SM the register budget is sized for
  static constexpr int kMinCtas = D == 64 ? 3 : (G <= 4 ? 2 : 1);
  // one split piece of another CTA (G heads of acc[D], max, sum, pad), fetched ahead
  // of this CTA's final merge -- where kMinCtas CTAs still fit the SM's 228 KB
  static constexpr int kPreOffset = (kIdsOffset + 2 * kIdWindow * 8 * 4 + 15) & ~15;
  static constexpr int kPieceBytes = G * (D + 4) * 4;
  static constexpr int kCtrlBytes = 80;
  static constexpr bool kPreFits =
      (1024 + kPreOffset + kPieceBytes + kCtrlBytes + 1024) * kMinCtas <= 228 * 1024;
  static constexpr int kPreBytes = kPreFits ? kPieceBytes : 0;
  static constexpr int kCtrlOffset = kPreOffset + kPreBytes;
  // after the control words (W, x0, x1, abort, last): the metadata barriers, then
  // the hand-off word of the fetched piece
  static constexpr int kMetaBarOffset = kCtrlOffset + 32;
  static_assert(kStages * 8 <= 32, "metadata barriers fit the control area");
  static constexpr int kPreStateOffset = kCtrlOffset + 64;
  static constexpr int kBytes = 1024 + kCtrlOffset + kCtrlBytes;  // + slack to align the ring to 1 KB
};

// The CTA owning global tile x when W tiles are split evenly over n CTAs
// (CTA c owns [c*W/n, (c+1)*W/n)): the c with c*W < (x+1)*n <= (c+1)*W. An fp32
// quotient is within one of it and two 64-bit products settle it (a 64-bit integer
// division costs hundreds of cycles, and the flushes run these for every thread).
__device__ __forceinline__ int owner_cta(long long x, long long W, int n) {
  const long long v = (x + 1) * n;
  int c = (int)((float)v / (float)W);
  while (c > 0 && (long long)c * W >= v) --c;
  while ((long long)(c + 1) * W < v) ++c;
  return c;
}

// Whether CTA c owns any tile (with more CTAs than tiles some own none; with at
// least as many tiles as CTAs every CTA owns floor(W/n) or more).
__device__ __forceinline__ bool cta_has_tiles(int c, long long W, int n) {
  return W >= n || (long long)c * W / n < (long long)(c + 1) * W / n;
}

__device__ __forceinline__ int clamp_len(int len, int cap, int max_len, bool &bad) {
  if (len < 0 || len > cap || len > max_len) {
    bad = true;
    return len < 0 ? 0 : min(min(len, cap), max_len);
  }
  return len;
}

// How the even-split kernel sees sequence b. With kWindow (a sliding window of
// `window` positions), from the block holding its first attended position on:
// its length shorter by `shift` whole blocks, its table read `shift` entries
// further on, and the `skip` positions of that first block that precede the
// window masked (skip < block_size <= 64: they lie in the first tile). Every place
// that counts tiles or reads the table takes lengths from here, so the CTA ranges,
// the producers' walks and the merges' owner arithmetic agree.
struct SeqView {
  int len, shift, skip;
};
template <bool kWindow>
__device__ __forceinline__ SeqView seq_view(int raw_len, int cap, int max_len, int window, int bs,
                                            bool &bad) {
  SeqView v;
  v.len = clamp_len(raw_len, cap, max_len, bad);
  v.shift = 0;
  v.skip = 0;
  if (kWindow) {
    const int lo = window_lo(v.len, window);
    v.shift = lo / bs;
    v.skip = lo - v.shift * bs;
    v.len -= v.shift * bs;
  }
  return v;
}

// tiles of one (sequence, kv head) segment; an empty sequence still gets one
// (empty) tile so that its output is written (zeros)
// floats per stored piece of one head: acc[D], max, sum and padding that keeps
// every piece 16-byte aligned for vector access
template <int D>
__host__ __device__ constexpr int piece_stride() { return D + 4; }

__device__ __forceinline__ int seg_tiles(int len) { return len > 0 ? (len + kTile - 1) / kTile : 1; }

// kWindow: a sliding window of p.window positions; every sequence is seen from
// the block holding its first attended position on (seq_view), and the first
// tile of each may start with positions before the window, which are masked (a
// separate instantiation, so that plain decode carries none of it)
template <typename T, int D, int G, bool kWindow>
__global__ void __launch_bounds__(kThreads, (Cfg<D, G>::kMinCtas))
    pa_decode_stream_kernel(const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using C = Cfg<D, G>;
  constexpr int NS = C::kStages;
  constexpr int KSTEPS = D / 16;
  constexpr int kPieceStride = piece_stride<D>();

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
  uint64_t *empty_bar = full_bar + NS;
  // meta_bar[s]: the tile's metadata is in meta[s] (one arrival per tile, even
  // when the stage's data copies are not issued); the consumers take the metadata
  // through it after a give-up, so they never read metadata not yet written.
  uint64_t *meta_bar = reinterpret_cast<uint64_t *>(smem + C::kMetaBarOffset);
  TileMeta *meta = reinterpret_cast<TileMeta *>(smem + C::kMetaOffset);
  float *mlbuf = reinterpret_cast<float *>(smem + C::kMlOffset);
  float *red = reinterpret_cast<float *>(smem + C::kRedOffset);
  long long *ctrl = reinterpret_cast<long long *>(smem + C::kCtrlOffset);  // W, x0, x1
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 3);
  volatile int *last_flag = abort_flag + 1;
  // the piece fetched ahead of the final merge: pre_state 0 = open, 1 = the producer
  // has issued its copy into pre_piece (landing on pre_bar), 2 = the consumers went
  // ahead without it, 3 = the producer found it not out yet (whichever sets it first
  // from 0 wins)
  int *pre_state = reinterpret_cast<int *>(smem + C::kPreStateOffset);
  uint64_t *pre_bar = reinterpret_cast<uint64_t *>(smem + C::kPreStateOffset + 8);
  const float *pre_piece = reinterpret_cast<const float *>(smem + C::kPreOffset);
  const uint32_t ring = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, nctas = p.grid_ctas;
  const int Hkv = p.num_kv_heads, B = p.num_seqs, bs = p.block_size;
  const int cap = p.max_blocks_per_seq * bs;

  // ---- size the whole job (every CTA does the same scan) and take an even share;
  // the lengths of up to 32 * kScanLoads sequences are loaded per round trip
  if (warp == kWarps) {
    long long W = 0;
    bool bad = false;
    for (int base = 0; base < B; base += 32 * kScanLoads) {
      int len[kScanLoads];
#pragma unroll
      for (int k = 0; k < kScanLoads; ++k) {
        const int bb = base + 32 * k + lane;
        len[k] = bb < B ? __ldg(p.context_lens + bb) : 0;
      }
      int tiles = 0;
#pragma unroll
      for (int k = 0; k < kScanLoads; ++k)
        if (base + 32 * k + lane < B)
          tiles += Hkv * seg_tiles(
                             seq_view<kWindow>(len[k], cap, p.max_context_len, p.window, bs, bad).len);
      for (int off = 16; off >= 1; off >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, off);
      W += tiles;
    }
    if (__any_sync(0xffffffffu, bad) && cta == 0 && lane == 0)
      atomicOr(&g_decode_error, PA_DEVERR_CONTEXT_LEN);
    if (lane == 0) {
      ctrl[0] = W;
      ctrl[1] = (long long)cta * W / nctas;
      ctrl[2] = (long long)(cta + 1) * W / nctas;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kWarps);
      mbar_init(&meta_bar[s], 1);
    }
    *abort_flag = 0;
    *pre_state = 0;
    mbar_init(pre_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const long long W = ctrl[0], x0 = ctrl[1], x1 = ctrl[2];
  if (x0 >= x1) return;  // nothing for this CTA (uniform)
  const int ntiles = (int)(x1 - x0);

  if (warp >= kWarps) {
    // ==================================================================== producers
    const bool v_producer = warp == kWarps + 1;
    // find the segment holding tile x0: sequences in order, kv heads inner
    long long pre = 0;
    int b = 0;
    bool bad = false;
    for (int base = 0; base < B; base += 32) {
      int tiles = 0;
      if (base + lane < B)
        tiles = Hkv * seg_tiles(seq_view<kWindow>(__ldg(p.context_lens + base + lane), cap,
                                                  p.max_context_len, p.window, bs, bad)
                                    .len);
      int incl = tiles;
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (pre + total > x0) {
        const unsigned hit = __ballot_sync(0xffffffffu, base + lane < B && pre + incl > x0);
        const int first = __ffs(hit) - 1;
        const int before = __shfl_sync(0xffffffffu, incl - tiles, first);
        b = base + first;
        pre += before;
        break;
      }
      pre += total;
    }
    SeqView view_b =
        seq_view<kWindow>(__ldg(p.context_lens + b), cap, p.max_context_len, p.window, bs, bad);
    int len_b = view_b.len, skip_b = view_b.skip;
    // the next sequence's length, loaded ahead of need
    int len_next = b + 1 < B ? __ldg(p.context_lens + b + 1) : 0;
    const bool fused = p.new_slots != nullptr;
    long long slot_b = fused ? __ldg(p.new_slots + b) : -1;
    long long slot_next = fused && b + 1 < B ? __ldg(p.new_slots + b + 1) : -1;
    int tb = seg_tiles(len_b);
    int kvh = (int)(x0 - pre) / tb;  // (x0 - pre < Hkv * tb: 32-bit division)
    int j = (int)(x0 - pre) % tb;
    const int box_rows = bs < kTile ? bs : kTile;
    const uint32_t box_bytes = 2u * C::kPanels * box_rows * 128u;
    const int32_t *tables = p.block_tables;
    // boxes of the tile at (b, j) and this lane's block id for it (issued one tile
    // ahead so the load overlaps the wait for a free stage)
    auto tile_boxes = [&](int jj, int len) {
      const int t0 = jj * kTile;
      const int nv = max(0, min(kTile, len - t0));
      return nv > 0 ? (bs <= kTile ? (t0 + nv - 1) / bs - t0 / bs + 1 : 1) : 0;
    };
    // Block ids travel through a window of kIdWindow tiles in shared memory, filled
    // by non-blocking copies kIdWindow tiles ahead of use: the tables are mostly
    // out of L2 (the K/V stream evicts them), so each id load costs a full HBM
    // round trip that must overlap the copies of the tiles before it.
    const uint32_t ids = smem_u32(smem + C::kIdsOffset) + (v_producer ? kIdWindow * 8 * 4 : 0);
    // cursor of the tile being fetched (ashift: its sequence's table shift)
    int ab = b, akvh = kvh, aj = j, alen = len_b, atb = tb, ashift = view_b.shift;
    auto fetch_ids = [&](int slot) {
      if (lane < tile_boxes(aj, alen))
        cp_async_4(ids + (slot * 8 + lane) * 4,
                   tables + (size_t)ab * p.max_blocks_per_seq + ashift + (aj * kTile) / bs + lane);
      cp_async_commit();
    };
    auto advance_ahead = [&]() {
      if (++aj == atb) {
        aj = 0;
        if (++akvh == Hkv) {
          akvh = 0;
          if (++ab < B) {
            const SeqView v = seq_view<kWindow>(__ldg(p.context_lens + ab), cap,
                                                p.max_context_len, p.window, bs, bad);
            alen = v.len;
            ashift = v.shift;
            atb = seg_tiles(alen);
          }
        }
      }
    };
    for (int k = 0; k < kIdWindow; ++k) {
      if (k < ntiles) {
        fetch_ids(k);
        if (k + 1 < ntiles) advance_ahead();
      } else {
        cp_async_commit();  // keep one group per tile
      }
    }
    int phys = -1;
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)));
    }
    // Everything above read only the lengths, the block tables and the slots.
    // Launched as a programmatic dependent (pa_decode_append_overlapped), the
    // kernel may have started before the preceding kernel finished: wait for it
    // here, before the first read of q, the new rows or the pools (no-op
    // otherwise), then let the next kernel start its own prologue.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the copies of the last NS tiles this warp issued (bit k: tile ntiles - NS + k)
    uint32_t issued_mask = 0;
    // The segment this CTA ends in may start here and go on in the next CTAs, which
    // make its other pieces at the start of theirs. With exactly one other piece, the
    // K producer, once its last copies are issued (the consumers still have the
    // tiles in the ring to go), checks the segment's counter and, if that piece is
    // out, copies it into shared memory: the final merge then reads no global
    // memory. (pre_cta: the CTA of that piece)
    int pre_cta = -1;
    bool pre_issued = false;
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % NS;
      // stage free? The consumers arrive once per tile whatever happened; after a
      // give-up this wait carries on without the early exit, so the producer never
      // runs a full ring ahead and never rewrites metadata the consumers may still
      // read
      if (i >= NS && !mbar_wait_bounded(&empty_bar[s], ((i / NS) & 1) ^ 1, abort_flag))
        mbar_wait_sure(&empty_bar[s], ((i / NS) & 1) ^ 1);
      // has any wait given up? (read after the free-stage wait, which orders it after
      // the consumers' give-up; used once the ids are in)
      const int gave_up = *abort_flag;
      // this tile's ids have landed once at most kIdWindow - 1 newer groups are pending
      cp_async_wait<kIdWindow - 1>();
      __syncwarp();
      phys = lane < tile_boxes(j, len_b)
                 ? reinterpret_cast<const int *>(smem + C::kIdsOffset +
                                                 (v_producer ? kIdWindow * 8 * 4 : 0))[(i % kIdWindow) * 8 + lane]
                 : -1;
      const int t0 = j * kTile;
      const int nvalid = max(0, min(kTile, len_b - t0));
      const bool seg_begin = (j == 0) || (i == 0);
      const bool seg_end = (j == tb - 1) || (i == ntiles - 1);
      const bool new_tok = fused && j == tb - 1 && len_b > 0;  // tile of position len - 1
      if (C::kPreBytes > 0 && !v_producer && j == 0 && x0 + i + tb > x1 && !p.starve) {
        const int cb = owner_cta(x0 + i + tb - 1, W, nctas);
        int n_other = 0, c_other = -1;
        for (int cc = cta + 1; cc <= cb && n_other < 2; ++cc)
          if (cta_has_tiles(cc, W, nctas)) {
            ++n_other;
            c_other = cc;
          }
        if (n_other == 1) pre_cta = c_other;
      }
      const bool ok = lane < tile_boxes(j, len_b) && phys >= 0 && phys < p.num_blocks;
      if (lane < tile_boxes(j, len_b) && !ok && !v_producer)
        atomicOr(&g_decode_error, PA_DEVERR_BLOCK_ID);
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      // copies go out only while nothing has given up (and never in the test mode):
      // a stage whose data never landed is not armed a second time
      const bool issue = !p.starve && !__any_sync(0xffffffffu, gave_up);
      issued_mask = (issued_mask >> 1) | (issue ? 1u << (NS - 1) : 0u);
      if (lane == 0 && !v_producer) {
        TileMeta &m = meta[s];
        m.b = b;
        m.kvh = kvh;
        m.j = j;
        m.seg_tiles = tb;
        m.nvalid = nvalid;
        m.seg_first_x = (int)(x0 + i - j);
        m.flags = (seg_begin ? 1 : 0) | (seg_end ? 2 : 0) | (new_tok ? 4 : 0);
        m.nskip = (kWindow && j == 0) ? min(skip_b, kTile - 1) : 0;
        m.new_slot = slot_b;
        if (issue)
          mbar_expect_tx_arrive(&full_bar[s], __popc(okmask) * box_bytes +
                                                  (seg_begin ? (uint32_t)C::kQBytes : 0u) +
                                                  (new_tok ? (uint32_t)C::kNewBytes : 0u));
        mbar_arrive(&meta_bar[s]);
      }
      __syncwarp();
      const uint32_t stage = ring + s * C::kStageBytes;
      {
        // one copy per lane: (box, panel) of this producer's operand (K or V)
        const int box = lane / C::kPanels;
        const int which = v_producer ? 1 : 0;
        const int pn = lane % C::kPanels;
        const int box_phys = __shfl_sync(0xffffffffu, phys, box & 31);
        const bool box_ok = box < 32 && ((okmask >> (box & 31)) & 1u);
        if (box_ok && issue) {
          // box of block t0/bs + box: whole block (bs <= 64) or a 64-row slice (bs > 64)
          const int r0 = bs > kTile ? t0 % bs : 0;
          const int row = bs > kTile ? 0 : box * bs;
          const int y = (box_phys * Hkv + kvh) * bs + r0;
          tma_load_2d(stage + (which * C::kPanels + pn) * kPanelBytes + row * 128,
                      which ? &tmap_v : &tmap_k, pn * 64, y, &full_bar[s]);
        }
      }
      if (lane == 0 && seg_begin && !v_producer && issue)
        bulk_g2s(smem + C::kQOffset + s * C::kQBytes,
                 static_cast<const T *>(p.q) + ((size_t)b * p.num_q_heads + (size_t)kvh * G) * D,
                 C::kQBytes, &full_bar[s]);
      if (lane == 0 && new_tok && !v_producer && issue) {
        const size_t row = ((size_t)b * Hkv + kvh) * D;
        unsigned char *dst = smem + C::kNewOffset + s * C::kNewBytes;
        bulk_g2s(dst, static_cast<const T *>(p.k_new) + row, D * 2, &full_bar[s]);
        bulk_g2s(dst + D * 2, static_cast<const T *>(p.v_new) + row, D * 2, &full_bar[s]);
      }
      // next tile: kv heads inner, then sequences
      if (i + 1 < ntiles) {
        if (++j == tb) {
          j = 0;
          if (++kvh == Hkv) {
            kvh = 0;
            ++b;
            const SeqView v =
                seq_view<kWindow>(len_next, cap, p.max_context_len, p.window, bs, bad);
            len_b = v.len;
            skip_b = v.skip;
            tb = seg_tiles(len_b);
            len_next = b + 1 < B ? __ldg(p.context_lens + b + 1) : 0;
            slot_b = slot_next;
            slot_next = fused && b + 1 < B ? __ldg(p.new_slots + b + 1) : -1;
          }
        }
      }
      // refill the window slot just used with the ids of tile i + kIdWindow
      if (i + kIdWindow < ntiles) {
        fetch_ids(i % kIdWindow);
        if (i + kIdWindow + 1 < ntiles) advance_ahead();
      } else {
        cp_async_commit();
      }
    }
    if (pre_cta >= 0) {
      // the counter counts the other pieces out; only this CTA's merge resets it
      const bool out = ld_acquire_gpu(p.ws_counters + cta) == 1;
      if (lane == 0 && atomicCAS(pre_state, 0, out ? 1 : 3) == 0 && out) {
        pre_issued = true;
        asm volatile("fence.proxy.async.global;" ::: "memory");  // the copy reads what was acquired
        mbar_expect_tx_arrive(pre_bar, (uint32_t)C::kPreBytes);
        bulk_g2s(smem + C::kPreOffset, p.ws_pieces + (size_t)(2 * pre_cta) * G * kPieceStride,
                 (uint32_t)C::kPreBytes, pre_bar);
      }
    }
    // the piece's copy, like the tiles', lands before the CTA exits
    if (pre_issued && lane == 0) {
      const unsigned long long t_start = global_ns();
      while (!mbar_try_wait(pre_bar, 0)) {
        if (global_ns() - t_start > kWaitLimitNs) {
          atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
          break;
        }
      }
    }
    // do not leave while copies may still land in this CTA's shared memory
    if (lane == 0) {
      for (int i = max(0, ntiles - NS); i < ntiles; ++i) {
        if (!((issued_mask >> (i - (ntiles - NS))) & 1u)) continue;  // nothing issued there
        const int s = i % NS;
        const unsigned long long t_start = global_ns();
        while (!mbar_try_wait(&full_bar[s], (i / NS) & 1)) {
          if (global_ns() - t_start > kWaitLimitNs) {
            atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
            break;
          }
        }
      }
    }
    return;
  }

  // ======================================================================= consumers
  // (their bounded waits start once the preceding kernel is done: see the producer)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int g = lane >> 2;  // fragment row group
  const int t = lane & 3;   // this lane's heads are 2t and 2t+1
  const int wrow = warp * 16;
  const int ld_row_k = wrow + (lane & 7) + 8 * ((lane >> 3) & 1);
  const int ld_chk_k = lane >> 4;
  const int ld_row_v = wrow + (lane & 7) + 8 * (lane >> 4);
  const int ld_chk_v = (lane >> 3) & 1;

  uint32_t qb[KSTEPS][2];
  float o[KSTEPS][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool gave_up = false;  // a data wait of this warp has failed

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % NS;
    // after a give-up the loop runs on (on whatever the stage holds) so every
    // consumer warp reaches every barrier below. A give-up leaves data barriers'
    // phases behind: a stage that is not armed again never completes, and a parity
    // wait on it then reports the older phase as done. Such a stale success can
    // only come after this warp's own wait on that stage failed (every warp waits
    // on every tile in order), so once this warp has seen a failed wait no data
    // wait counts as landed, and the metadata comes through its own barrier, which
    // completes once per tile whatever happened: all warps read the same, fully
    // written metadata. Until then a landed stage carries its metadata (written
    // before the producer's arrival).
    const bool ok = __all_sync(
        0xffffffffu, mbar_wait_bounded(&full_bar[s], (i / NS) & 1, abort_flag, p.wait_ns));
    const bool landed = ok && !gave_up;
    if (!landed) {
      gave_up = true;
      mbar_wait_sure(&meta_bar[s], (i / NS) & 1);
    }
    __syncwarp();
    const TileMeta mt = meta[s];
    const uint32_t kst = ring + s * C::kStageBytes;
    const uint32_t vst = kst + C::kPanels * kPanelBytes;
    if (mt.flags & 1) {
      // a new segment piece: reset the state and take its q rows (Q^T as the B operand)
      const uint32_t *qs =
          reinterpret_cast<const uint32_t *>(smem + C::kQOffset + s * C::kQBytes);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        qb[kk][0] = g < G ? qs[(g * D + kk * 16 + 2 * t) / 2] : 0u;
        qb[kk][1] = g < G ? qs[(g * D + kk * 16 + 8 + 2 * t) / 2] : 0u;
      }
#pragma unroll
      for (int x = 0; x < KSTEPS; ++x) o[x][0] = o[x][1] = o[x][2] = o[x][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }
    const int nvalid = mt.nvalid;
    const int nskip = kWindow ? mt.nskip : 0;
    if ((mt.flags & 4) && landed && (nvalid - 1) / 16 == warp) {
      // fused write: the new token (last valid row) replaces what the cache held
      // in this tile, and is stored at its slot for later steps (not after a
      // give-up: the copied rows may not have landed)
      constexpr int kChunks = D / 8;  // 16-byte chunks per row
      const int r = nvalid - 1;
      if (lane < 2 * kChunks) {
        const int which = lane / kChunks, c = lane % kChunks;  // which: 0 = K, 1 = V
        const uint4 v = *reinterpret_cast<const uint4 *>(smem + C::kNewOffset +
                                                         s * C::kNewBytes + which * D * 2 + c * 16);
        unsigned char *panel = smem + s * C::kStageBytes + (which * C::kPanels + c / 8) * kPanelBytes;
        *reinterpret_cast<uint4 *>(panel + r * 128 + (((c % 8) ^ (r & 7)) << 4)) = v;
        const long long slot = mt.new_slot;
        if (slot >= 0 && slot < (long long)p.num_blocks * bs) {
          const long long blk = slot / bs, off = slot - blk * bs;
          unsigned char *cache = static_cast<unsigned char *>(which ? p.v_cache_w : p.k_cache_w);
          *reinterpret_cast<uint4 *>(cache + (((size_t)blk * Hkv + mt.kvh) * bs + off) * D * 2 +
                                     c * 16) = v;
        } else if (slot >= 0 && lane == 0) {
          atomicOr(&g_decode_error, PA_DEVERR_SLOT);
        }
      }
      __syncwarp();
    }
    if (nvalid < wrow + 16 || nskip > wrow) {
      // rows past the valid tokens, or before a sliding window, may hold anything
      // (0 * NaN would poison the product): zero this warp's own V rows there
      // before reading them
      unsigned char *vz = smem + s * C::kStageBytes + C::kPanels * kPanelBytes;
      for (int r = (kWindow ? wrow : max(nvalid, wrow)) + (lane >> 3); r < wrow + 16; r += 4) {
        if (kWindow && r < nvalid && r >= nskip) continue;
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          *reinterpret_cast<uint4 *>(vz + pn * kPanelBytes + r * 128 + (lane & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }

    // ---- S^T[16 tokens][8 heads] = K . Q^T
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KSTEPS; kk += 2) {
      uint32_t a[4], a2[4];
      ldsm_x4(swz(kst + (kk / 4) * kPanelBytes, ld_row_k, 2 * (kk % 4) + ld_chk_k), a);
      ldsm_x4(swz(kst + ((kk + 1) / 4) * kPanelBytes, ld_row_k, 2 * ((kk + 1) % 4) + ld_chk_k),
              a2);
      Mma<T>::run(sa, a, qb[kk][0], qb[kk][1]);
      Mma<T>::run(sb, a2, qb[kk + 1][0], qb[kk + 1][1]);
    }
    const bool va = wrow + g < nvalid && wrow + g >= nskip;
    const bool vb = wrow + g + 8 < nvalid && wrow + g + 8 >= nskip;
    const float s0 = va ? (sa[0] + sb[0]) * p.scale_log2 : -INFINITY;
    const float s1 = va ? (sa[1] + sb[1]) * p.scale_log2 : -INFINITY;
    const float s2 = vb ? (sa[2] + sb[2]) * p.scale_log2 : -INFINITY;
    const float s3 = vb ? (sa[3] + sb[3]) * p.scale_log2 : -INFINITY;

    // ---- online softmax over the warp's 16 tokens (max shared by a column's 8 lanes)
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float r0, r1, r2, r3;
    const uint32_t x0w = Mma<T>::pack(s0 == -INFINITY ? 0.f : exp2f(s0 - mn0),
                                      s1 == -INFINITY ? 0.f : exp2f(s1 - mn1), r0, r1);
    const uint32_t x1w = Mma<T>::pack(s2 == -INFINITY ? 0.f : exp2f(s2 - mn0),
                                      s3 == -INFINITY ? 0.f : exp2f(s3 - mn1), r2, r3);
    l0 = l0 * al0 + (r0 + r2);
    l1 = l1 * al1 + (r1 + r3);
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int x = 0; x < KSTEPS; ++x) {
        o[x][0] *= al0;
        o[x][1] *= al1;
        o[x][2] *= al0;
        o[x][3] *= al1;
      }
    }
    const uint32_t pb0 = movmatrix_trans(x0w);
    const uint32_t pb1 = movmatrix_trans(x1w);

    // ---- O^T[d][heads] += V^T[d][tokens] . P[tokens][heads]
#pragma unroll
    for (int x = 0; x < KSTEPS; ++x) {
      uint32_t a[4];
      ldsm_x4_trans(swz(vst + (x / 4) * kPanelBytes, ld_row_v, 2 * (x % 4) + ld_chk_v), a);
      Mma<T>::run(o[x], a, pb0, pb1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);

    if (!(mt.flags & 2)) continue;
    // ================================= end of this CTA's piece of the segment: flush
    float sl0 = l0, sl1 = l1;
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
      sl0 += __shfl_xor_sync(0xffffffffu, sl0, off);
      sl1 += __shfl_xor_sync(0xffffffffu, sl1, off);
    }
    if (g == 0) {
      mlbuf[(warp * 8 + 2 * t) * 2] = m0;
      mlbuf[(warp * 8 + 2 * t) * 2 + 1] = sl0;
      mlbuf[(warp * 8 + 2 * t + 1) * 2] = m1;
      mlbuf[(warp * 8 + 2 * t + 1) * 2 + 1] = sl1;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
    {
      const int h0 = 2 * t, h1 = 2 * t + 1;
      float f0 = 0.f, f1 = 0.f;
      if (h0 < G) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mlbuf[(w * 8 + h0) * 2]);
        f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
      }
      if (h1 < G) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mlbuf[(w * 8 + h1) * 2]);
        f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
      }
#pragma unroll
      for (int x = 0; x < KSTEPS; ++x) {
        const int d = x * 16 + g;
        if (h0 < G) {
          red[(warp * G + h0) * D + d] = o[x][0] * f0;
          red[(warp * G + h0) * D + d + 8] = o[x][2] * f0;
        }
        if (h1 < G) {
          red[(warp * G + h1) * D + d] = o[x][1] * f1;
          red[(warp * G + h1) * D + d + 8] = o[x][3] * f1;
        }
      }
    }
    const bool whole = mt.seg_first_x >= x0 && (long long)mt.seg_first_x + mt.seg_tiles <= x1;
    const bool first_of_cta = mt.seg_first_x <= x0;
    const int slot = first_of_cta ? 2 * cta : 2 * cta + 1;
    const size_t hq_base = (size_t)mt.b * p.num_q_heads + (size_t)mt.kvh * G;
    // a split segment's pieces belong to CTAs ca..cb (those of them that own tiles)
    const long long sf = mt.seg_first_x;
    const int ca = owner_cta(sf, W, nctas);
    const int cb = owner_cta(sf + mt.seg_tiles - 1, W, nctas);
    // The CTA holding the segment's first tiles reaches this point at the end of its
    // range, when the other pieces (made at the start of theirs) are normally out
    // already: if the counter says so, it merges at once from its own values and
    // theirs, without writing its piece, fencing or counting (same order and
    // arithmetic as the merge below, so the same bits)
    // (from shared memory when the producer has fetched the other piece already)
    if (!whole && ca == cta && tid == 0) {
      int pieces = 0;
      for (int cc = ca; cc <= cb; ++cc) pieces += cta_has_tiles(cc, W, nctas) ? 1 : 0;
      int flag = 0;
      if (C::kPreBytes > 0 && pieces == 2 && !p.starve) {
        // the producer decides one counter read after its last issue: wait for
        // that (briefly), then take the piece from shared memory if it copied it
        const unsigned long long t_start = global_ns();
        while (*reinterpret_cast<volatile int *>(pre_state) == 0 && !*abort_flag &&
               global_ns() - t_start < kPreWaitNs) {
        }
        if (atomicCAS(pre_state, 0, 2) == 1 && mbar_wait_bounded(pre_bar, 0, abort_flag))
          flag = 3;
      }
      if (flag == 0) flag = ld_acquire_gpu(p.ws_counters + ca) == pieces - 1 ? 2 : 0;
      *last_flag = flag;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
    const bool from_smem = !whole && ca == cta && *last_flag == 3;
    const bool merge_now = !whole && ca == cta && (*last_flag == 2 || from_smem);
    if (merge_now && !from_smem) __threadfence();
    for (int e0 = tid * 4; e0 < G * D; e0 += kWarps * 32 * 4) {
      const int h = e0 / D, d = e0 % D;
      float M = -INFINITY;
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mlbuf[(w * 8 + h) * 2]);
      float L = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mlbuf[(w * 8 + h) * 2];
        if (mw != -INFINITY) L += exp2f(mw - M) * mlbuf[(w * 8 + h) * 2 + 1];
      }
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < kWarps; ++w) {
        const float4 v = *reinterpret_cast<const float4 *>(red + (w * G + h) * D + d);
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      if (whole) {
        const float inv = L > 0.f ? 1.f / L : 0.f;
        *reinterpret_cast<uint2 *>(static_cast<T *>(p.out) + (hq_base + h) * D + d) =
            Elem<T>::from_f32x4(sum.x * inv, sum.y * inv, sum.z * inv, sum.w * inv);
      } else if (merge_now) {
        // this CTA's piece (M, L, sum) first, then the others' in CTA order
        auto piece = [&](int cc) {
          return from_smem ? pre_piece + h * kPieceStride
                           : p.ws_pieces + ((size_t)(2 * cc) * G + h) * kPieceStride;
        };
        auto rd = [&](const float *a) { return from_smem ? *a : __ldcg(a); };
        auto rd4 = [&](const float *a) {
          return from_smem ? *reinterpret_cast<const float4 *>(a)
                           : __ldcg(reinterpret_cast<const float4 *>(a));
        };
        float Mm = M;
        for (int cc = ca + 1; cc <= cb; ++cc) {
          if (!cta_has_tiles(cc, W, nctas)) continue;
          Mm = fmaxf(Mm, rd(piece(cc) + D));
        }
        float Lm = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
          const float w = exp2f(M - Mm);
          Lm += w * L;
          acc.x += w * sum.x;
          acc.y += w * sum.y;
          acc.z += w * sum.z;
          acc.w += w * sum.w;
        }
        for (int cc = ca + 1; cc <= cb; ++cc) {
          if (!cta_has_tiles(cc, W, nctas)) continue;
          const float *pc = piece(cc);
          const float mc = rd(pc + D);
          if (mc == -INFINITY) continue;
          const float w = exp2f(mc - Mm);
          Lm += w * rd(pc + D + 1);
          const float4 v = rd4(pc + d);
          acc.x += w * v.x;
          acc.y += w * v.y;
          acc.z += w * v.z;
          acc.w += w * v.w;
        }
        const float inv = Lm > 0.f ? 1.f / Lm : 0.f;
        *reinterpret_cast<uint2 *>(static_cast<T *>(p.out) + (hq_base + h) * D + d) =
            Elem<T>::from_f32x4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      } else {
        float *pc = p.ws_pieces + ((size_t)slot * G + h) * kPieceStride;
        *reinterpret_cast<float4 *>(pc + d) = sum;
        if (d == 0) {
          pc[D] = M;
          pc[D + 1] = L;
        }
      }
    }
    if (merge_now) {
      // every other piece had arrived: nothing more counts on this segment
      if (tid == 0) p.ws_counters[ca] = 0;
    } else if (!whole) {
      // the piece is out; the CTA that completes the segment's last piece merges
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
      if (tid == 0) {
        int pieces = 0;  // one per CTA in [ca, cb] that owns tiles
        for (int cc = ca; cc <= cb; ++cc) pieces += cta_has_tiles(cc, W, nctas) ? 1 : 0;
        *last_flag = atomicAdd(p.ws_counters + ca, 1) == pieces - 1;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
      if (*last_flag) {
        __threadfence();
        const long long x0a = (long long)ca * W / nctas;
        for (int e0 = tid * 4; e0 < G * D; e0 += kWarps * 32 * 4) {
          const int h = e0 / D, d = e0 % D;
          float M = -INFINITY;
          for (int cc = ca; cc <= cb; ++cc) {
            if (!cta_has_tiles(cc, W, nctas)) continue;
            const int sl = (cc == ca && sf > x0a) ? 2 * cc + 1 : 2 * cc;
            M = fmaxf(M, __ldcg(p.ws_pieces + ((size_t)sl * G + h) * kPieceStride + D));
          }
          float L = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int cc = ca; cc <= cb; ++cc) {
            if (!cta_has_tiles(cc, W, nctas)) continue;
            const int sl = (cc == ca && sf > x0a) ? 2 * cc + 1 : 2 * cc;
            const float *pc = p.ws_pieces + ((size_t)sl * G + h) * kPieceStride;
            const float mc = __ldcg(pc + D);
            if (mc == -INFINITY) continue;
            const float w = exp2f(mc - M);
            L += w * __ldcg(pc + D + 1);
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(pc + d));
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          *reinterpret_cast<uint2 *>(static_cast<T *>(p.out) + (hq_base + h) * D + d) =
              Elem<T>::from_f32x4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
        if (tid == 0) p.ws_counters[ca] = 0;  // every piece has arrived: ready for the next call
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");  // red / mlbuf reused next
  }
}
}  // namespace tc

// ------------------------------------------------------------------------------ merge kernel
// One CTA per (q head, sequence), one thread per output element: combine the
// partitions' (max, sum, weighted V) states by log-sum-exp.
template <typename T, int D>
__global__ void __launch_bounds__(D) pa_decode_merge_kernel(
    void *out_, const float *__restrict__ ws_acc, const float *__restrict__ ws_ml,
    const int32_t *__restrict__ context_lens, int num_q_heads, int partition_tokens,
    int max_parts, int max_context_len, int cap, int window) {
  const int hqi = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  int len = __ldg(context_lens + b);
  len = len < 0 ? 0 : min(min(len, cap), max_context_len);
  const int nparts = (len - window_lo(len, window) + partition_tokens - 1) / partition_tokens;
  if (nparts <= 1) return;  // written by the partition kernel
  const size_t hq = (size_t)b * num_q_heads + hqi;
  const float *ml = ws_ml + hq * max_parts * 2;
  float M = -INFINITY;
  for (int i = 0; i < nparts; ++i) M = fmaxf(M, ml[2 * i]);
  float Ls = 0.f, acc = 0.f;
  for (int i = 0; i < nparts; ++i) {
    const float w = exp2f(ml[2 * i] - M);
    Ls += w * ml[2 * i + 1];
    acc += w * ws_acc[(hq * max_parts + i) * D + d];
  }
  T *out = static_cast<T *>(out_);
  out[hq * D + d] = Elem<T>::from_f32(acc / Ls);
}

}  // namespace

// ================================================================================ host side
namespace {

constexpr int kMaxDevices = 64;
constexpr int kPartitionQuantum = 64;   // partitions are whole tiles for every head_dim
constexpr int kMaxPartitionTokens = 8192;
constexpr int kSmCount = 148;
constexpr int kCtasPerSm = 3;

// ---- TMA tensor maps over a pool viewed as [num_blocks * num_kv_heads * block_size rows][D]
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

struct TmapKey {
  const void *base;
  long long rows;
  int head_dim, box_rows, dtype;
  bool operator==(const TmapKey &o) const {
    return base == o.base && rows == o.rows && head_dim == o.head_dim && box_rows == o.box_rows &&
           dtype == o.dtype;
  }
};

// Encoding costs a few microseconds; the same pools come back call after call.
bool pool_tensor_map(CUtensorMap *map, const void *base, long long rows, int head_dim,
                     int box_rows, pa_dtype dtype) {
  constexpr int kSlots = 16;
  static std::mutex mu;
  static TmapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static int used = 0, next = 0;
  const TmapKey key{base, rows, head_dim, box_rows, (int)dtype};
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (keys[i] == key) {
      *map = maps[i];
      return true;
    }
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  CUtensorMap m;
  if (enc(&m, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
          2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = used < kSlots ? used++ : (next++ % kSlots);
  keys[slot] = key;
  maps[slot] = m;
  *map = m;
  return true;
}

bool tensor_core_block_size(int bs) { return bs >= 8 && (bs & (bs - 1)) == 0; }

template <typename Kernel>
bool ensure_smem(Kernel kernel, size_t smem, size_t (&configured)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (smem > configured[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return false;
    configured[dev] = smem;
  }
  return true;
}

// Bytes at the start of every workspace that hold the even-split kernel's
// counters; they must be zero before the first call and every call leaves them
// zero. The split-partition scratch of the SIMT path starts after them.
constexpr size_t kCounterRegion = kPaCounterRegionBytes;
constexpr int kMaxStreamCtas = (int)(kCounterRegion / sizeof(int));

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return kSmCount;
  return n;
}

template <int D, int G>
int stream_ctas_per_sm() {
  static int per_sm[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  if (!per_sm[dev]) {
    auto kernel = tc::pa_decode_stream_kernel<__nv_bfloat16, D, G, false>;
    const size_t smem = tc::Cfg<D, G>::kBytes;
    int n = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, tc::kThreads, smem) !=
            cudaSuccess ||
        n <= 0)
      n = 1;
    per_sm[dev] = n;
  }
  return per_sm[dev];
}

template <int D>
int stream_ctas_per_sm_g(int group) {
  switch (group) {
    case 2: return stream_ctas_per_sm<D, 2>();
    case 4: return stream_ctas_per_sm<D, 4>();
    default: return stream_ctas_per_sm<D, 8>();
  }
}

// CTAs of the even-split kernel: one resident wave by default; with
// partition_tokens > 0, about partition_tokens tokens of one kv head per CTA.
int stream_grid(int num_seqs, int num_kv_heads, int group, int head_dim, int max_context_len,
                int partition_tokens) {
  long long n;
  if (partition_tokens > 0) {
    const long long tiles = (long long)num_seqs * num_kv_heads *
                            std::max(1, (max_context_len + 63) / 64);
    n = (tiles + partition_tokens / 64 - 1) / (partition_tokens / 64);
  } else {
    n = (long long)sm_count() *
        (head_dim == 128 ? stream_ctas_per_sm_g<128>(group) : stream_ctas_per_sm_g<64>(group));
  }
  return (int)std::max(1LL, std::min<long long>(n, kMaxStreamCtas));
}

bool uses_stream_kernel(int group, int block_size, int num_blocks, int num_kv_heads) {
  const long long rows = (long long)num_blocks * num_kv_heads * block_size;
  // one q head per kv head leaves 7/8 of the MMA N dimension idle: the SIMT
  // kernel measured faster there
  return group > 1 && tensor_core_block_size(block_size) && rows <= INT32_MAX;
}

// A sliding window runs on the even-split kernel when the positions of a
// block before the window fit in one 64-token tile; otherwise (and where the
// even-split kernel does not run at all) in the partition kernel.
bool window_on_stream(int group, int block_size, int num_blocks, int num_kv_heads) {
  return uses_stream_kernel(group, block_size, num_blocks, num_kv_heads) &&
         block_size <= tc::kTile;
}

size_t stream_workspace(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int max_context_len, int partition_tokens) {
  const int group = num_q_heads / num_kv_heads;
  const int n = stream_grid(num_seqs, num_kv_heads, group, head_dim, max_context_len,
                            partition_tokens);
  return (size_t)2 * n * group * (head_dim + 4) * sizeof(float);
}

template <typename T, int D, int G>
pa_status launch_decode(const DecodeParams &prm, int num_seqs, void *out, pa_dtype dtype,
                        cudaStream_t stream) {
  const bool win = prm.window > 0;
  if (win ? window_on_stream(G, prm.block_size, prm.num_blocks, prm.num_kv_heads)
          : uses_stream_kernel(G, prm.block_size, prm.num_blocks, prm.num_kv_heads)) {
    using C = tc::Cfg<D, G>;
    static size_t configured[kMaxDevices] = {};
    const long long rows = (long long)prm.num_blocks * prm.num_kv_heads * prm.block_size;
    const int box_rows = prm.block_size < tc::kTile ? prm.block_size : tc::kTile;
    CUtensorMap tk, tv;
    if (!pool_tensor_map(&tk, prm.k_cache, rows, D, box_rows, dtype) ||
        !pool_tensor_map(&tv, prm.v_cache, rows, D, box_rows, dtype))
      return PA_ERR_CUDA;
    static size_t configured_w[kMaxDevices] = {};
    if (!(win ? ensure_smem(tc::pa_decode_stream_kernel<T, D, G, true>, (size_t)C::kBytes,
                            configured_w)
              : ensure_smem(tc::pa_decode_stream_kernel<T, D, G, false>, (size_t)C::kBytes,
                            configured)))
      return PA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)prm.grid_ctas);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = C::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = prm.early_start ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e =
        win ? cudaLaunchKernelEx(&cfg, tc::pa_decode_stream_kernel<T, D, G, true>, tk, tv, prm)
            : cudaLaunchKernelEx(&cfg, tc::pa_decode_stream_kernel<T, D, G, false>, tk, tv, prm);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  using L = Smem<T, D, G>;
  static size_t configured[kMaxDevices] = {};
  const size_t smem = L::bytes(prm.table_slice);
  if (!ensure_smem(pa_decode_partition_kernel<T, D, G>, smem, configured)) return PA_ERR_CUDA;
  dim3 grid((unsigned)prm.max_parts, (unsigned)prm.num_kv_heads, (unsigned)num_seqs);
  pa_decode_partition_kernel<T, D, G><<<grid, kThreads, smem, stream>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (prm.max_parts > 1) {
    dim3 mgrid((unsigned)prm.num_q_heads, (unsigned)num_seqs);
    pa_decode_merge_kernel<T, D><<<mgrid, D, 0, stream>>>(
        out, prm.ws_acc, prm.ws_ml, prm.context_lens, prm.num_q_heads, prm.partition_tokens,
        prm.max_parts, prm.max_context_len, prm.max_blocks_per_seq * prm.block_size, prm.window);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <typename T, int D>
pa_status dispatch_group(int group, const DecodeParams &prm, int num_seqs, void *out,
                         pa_dtype dtype, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode<T, D, 1>(prm, num_seqs, out, dtype, stream);
    case 2: return launch_decode<T, D, 2>(prm, num_seqs, out, dtype, stream);
    case 4: return launch_decode<T, D, 4>(prm, num_seqs, out, dtype, stream);
    case 8: return launch_decode<T, D, 8>(prm, num_seqs, out, dtype, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <typename T>
pa_status dispatch_dim(int head_dim, int group, const DecodeParams &prm, int num_seqs, void *out,
                       pa_dtype dtype, cudaStream_t stream) {
  switch (head_dim) {
    case 64: return dispatch_group<T, 64>(group, prm, num_seqs, out, dtype, stream);
    case 128: return dispatch_group<T, 128>(group, prm, num_seqs, out, dtype, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}


int resolve_partition(int num_seqs, int num_kv_heads, int max_context_len, int requested) {
  if (requested > 0) return requested;
  return pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Test mode of the bounded waits (pa_debug_wait_test): read at every launch.
std::atomic<int> g_wait_test{0};
std::atomic<long long> g_wait_test_ns{0};

}  // namespace

extern "C" pa_status pa_debug_wait_test(int enable, long long consumer_wait_ns) {
  if (enable && (consumer_wait_ns <= 0 || consumer_wait_ns > (long long)kWaitLimitNs))
    return PA_ERR_INVALID;
  g_wait_test_ns.store(enable ? consumer_wait_ns : 0);
  g_wait_test.store(enable ? 1 : 0);
  return PA_OK;
}

extern "C" int pa_decode_default_partition(int num_seqs, int num_kv_heads, int max_context_len) {
  // Long enough to amortise the merge, short enough that the grid covers the
  // SMs several times over so uneven lengths balance out.
  const int round_up = ((max_context_len + kPartitionQuantum - 1) / kPartitionQuantum) *
                       kPartitionQuantum;
  int pt = 512;
  const long long pairs = (long long)num_seqs * num_kv_heads;
  while (pt > 128 && pairs * ((max_context_len + pt - 1) / pt) < 2LL * kSmCount * kCtasPerSm)
    pt /= 2;
  if (round_up > 0 && round_up < pt) pt = round_up;
  return pt < kPartitionQuantum ? kPartitionQuantum : pt;
}

size_t simt_workspace(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int max_context_len, int partition_tokens) {
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  const long long parts = (max_context_len + pt - 1) / pt;
  if (parts <= 1) return 0;
  return (size_t)num_seqs * num_q_heads * parts * (head_dim + 2) * sizeof(float);
}

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                           int head_dim, int max_context_len,
                                           int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_context_len <= 0 || partition_tokens < 0 || num_q_heads % num_kv_heads)
    return 0;
  // either kernel may run (it depends on the block size): size for the larger
  const size_t simt = simt_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                     max_context_len, partition_tokens);
  const int group = num_q_heads / num_kv_heads;
  // (the even-split kernel's pieces)
  const size_t stream = (group == 2 || group == 4 || group == 8) &&
                                (head_dim == 64 || head_dim == 128)
                            ? stream_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len, partition_tokens)
                            : 0;
  const size_t body = simt > stream ? simt : stream;
  return body ? kCounterRegion + body : 0;
}

extern "C" int pa_decode_grid_ctas(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, int max_context_len,
                                   int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      block_size <= 0 || num_blocks <= 0 || (head_dim != 64 && head_dim != 128) ||
      max_context_len < 0 || partition_tokens < 0 || partition_tokens % kPartitionQuantum)
    return 0;
  const int group = num_q_heads / num_kv_heads;
  if (!uses_stream_kernel(group, block_size, num_blocks, num_kv_heads)) return 0;
  return stream_grid(num_seqs, num_kv_heads, group, head_dim, max_context_len, partition_tokens);
}

extern "C" int pa_decode_launches(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, int max_context_len,
                                  int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      block_size <= 0 || num_blocks <= 0 || head_dim <= 0)
    return 0;
  const int group = num_q_heads / num_kv_heads;
  if (uses_stream_kernel(group, block_size, num_blocks, num_kv_heads)) return 1;
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  return max_context_len > pt ? 2 : 1;
}

namespace {

// Workspace one decode call needs (bytes, 0 for none), for the kernel that call
// runs: the even-split kernel's counters and pieces, or the
// partition kernel's partial states when the longest context has more than one
// partition. Arguments already validated.
size_t decode_need(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                   int num_blocks, int max_context_len, int partition_tokens, int window) {
  const int group = num_q_heads / num_kv_heads;
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  const int max_parts = max_context_len > 0 ? (max_context_len + pt - 1) / pt : 1;
  const bool wstream =
      window > 0 && window_on_stream(group, block_size, num_blocks, num_kv_heads);
  const bool streamk =
      (window == 0 && uses_stream_kernel(group, block_size, num_blocks, num_kv_heads)) || wstream;
  if (streamk) {
    const int nctas = stream_grid(num_seqs, num_kv_heads, group, head_dim, max_context_len,
                                  partition_tokens);
    return kCounterRegion + (size_t)2 * nctas * group * (head_dim + 4) * sizeof(float);
  }
  return max_parts > 1 ? kCounterRegion + (size_t)num_seqs * num_q_heads * max_parts *
                                              (head_dim + 2) * sizeof(float)
                       : 0;
}

// The new token of every sequence, written by the decode kernel itself.
struct FusedWrite {
  const void *k_new;
  const void *v_new;
  const int64_t *slots;
  void *k_cache;
  void *v_cache;
};

pa_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, int max_context_len, int num_seqs,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, float scale, pa_dtype dtype, void *workspace,
                      size_t workspace_bytes, int partition_tokens, void *stream,
                      const FusedWrite *fw, int window, bool early_start = false) {
  if (window < 0) return PA_ERR_INVALID;
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      (dtype != PA_F16 && dtype != PA_BF16))
    return PA_ERR_INVALID;
  if (partition_tokens < 0 || partition_tokens % kPartitionQuantum ||
      partition_tokens > kMaxPartitionTokens)
    return PA_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PA_ERR_INVALID;
  if ((long long)num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_INVALID;

  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PA_ERR_UNSUPPORTED;
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  const int max_parts = max_context_len > 0 ? (max_context_len + pt - 1) / pt : 1;
  // a sliding window runs on the even-split kernel (its kWindow instantiation)
  // where the block size allows (window_on_stream), else in the partition kernel
  const bool wstream =
      window > 0 && window_on_stream(group, block_size, num_blocks, num_kv_heads);
  const bool streamk = (window == 0 && uses_stream_kernel(group, block_size, num_blocks,
                                                          num_kv_heads)) ||
                       wstream;
  const int nctas = streamk ? stream_grid(num_seqs, num_kv_heads, group, head_dim,
                                          max_context_len, partition_tokens)
                            : 0;
  const size_t need = decode_need(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                  num_blocks, max_context_len, partition_tokens, window);
  if (need > workspace_bytes || (need && (!workspace || !aligned(workspace, 16))))
    return PA_ERR_INVALID;
  float *ws_body =
      need ? reinterpret_cast<float *>(static_cast<char *>(workspace) + kCounterRegion) : nullptr;

  DecodeParams prm;
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.ws_acc = streamk ? nullptr : ws_body;
  prm.ws_ml = (!streamk && need) ? ws_body + (size_t)num_seqs * num_q_heads * max_parts * head_dim
                                 : nullptr;
  prm.num_seqs = num_seqs;
  prm.grid_ctas = nctas;
  prm.ws_counters = streamk ? static_cast<int *>(workspace) : nullptr;
  prm.ws_pieces = streamk ? ws_body : nullptr;
  prm.k_new = fw ? fw->k_new : nullptr;
  prm.v_new = fw ? fw->v_new : nullptr;
  prm.new_slots = fw ? fw->slots : nullptr;
  prm.k_cache_w = fw ? fw->k_cache : nullptr;
  prm.v_cache_w = fw ? fw->v_cache : nullptr;
  prm.window = window;
  prm.early_start = early_start ? 1 : 0;
  prm.starve = g_wait_test.load();
  prm.wait_ns = prm.starve ? (unsigned long long)g_wait_test_ns.load() : kWaitLimitNs;
  if (fw && !streamk) return PA_ERR_INVALID;  // only the even-split kernel writes
  prm.max_blocks_per_seq = max_blocks_per_seq;
  prm.max_context_len = max_context_len;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition_tokens = pt;
  prm.max_parts = max_parts;
  prm.table_slice = pt / block_size + 2;
  prm.scale_log2 = scale * 1.4426950408889634f;
  if ((size_t)prm.table_slice * 4 > 16384) return PA_ERR_UNSUPPORTED;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PA_BF16)
    return dispatch_dim<__nv_bfloat16>(head_dim, group, prm, num_seqs, out, dtype, st);
  return dispatch_dim<__half>(head_dim, group, prm, num_seqs, out, dtype, st);
}

}  // namespace

extern "C" pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, int max_context_len, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, float scale, pa_dtype dtype, void *workspace,
                               size_t workspace_bytes, int partition_tokens, void *stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, scale, dtype, workspace, workspace_bytes, partition_tokens,
                     stream, nullptr, 0);
}

extern "C" pa_status pa_decode_window(void *out, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *context_lens,
                                      int max_context_len, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size,
                                      int num_blocks, float scale, int window, pa_dtype dtype,
                                      void *workspace, size_t workspace_bytes,
                                      int partition_tokens, void *stream) {
  if (window <= 0) return PA_ERR_INVALID;
  return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, scale, dtype, workspace, workspace_bytes, partition_tokens,
                     stream, nullptr, window);
}

extern "C" int pa_decode_window_launches(int num_seqs, int num_q_heads, int num_kv_heads,
                                         int head_dim, int block_size, int num_blocks,
                                         int max_context_len, int window,
                                         int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || window <= 0)
    return 0;
  // the even-split kernel
  if (window_on_stream(num_q_heads / num_kv_heads, block_size, num_blocks, num_kv_heads))
    return 1;
  // the partition kernel, and the merge kernel when the longest context has
  // more than one partition (partitions are sized from max_context_len)
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  return max_context_len > pt ? 2 : 1;
}

extern "C" int pa_decode_append_window_launches(int num_seqs, int num_q_heads, int num_kv_heads,
                                                int head_dim, int block_size, int num_blocks,
                                                int max_context_len, int window,
                                                int partition_tokens) {
  const int decode = pa_decode_window_launches(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               block_size, num_blocks, max_context_len, window,
                                               partition_tokens);
  if (decode == 0) return 0;
  // on the even-split kernel the write is fused; otherwise the write kernel runs first
  return window_on_stream(num_q_heads / num_kv_heads, block_size, num_blocks, num_kv_heads)
             ? decode
             : 1 + decode;
}

extern "C" int pa_decode_append_launches(int num_seqs, int num_q_heads, int num_kv_heads,
                                         int head_dim, int block_size, int num_blocks,
                                         int max_context_len, int partition_tokens) {
  const int decode = pa_decode_launches(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                        block_size, num_blocks, max_context_len,
                                        partition_tokens);
  if (decode == 0) return 0;
  const int group = num_q_heads / num_kv_heads;
  return uses_stream_kernel(group, block_size, num_blocks, num_kv_heads) ? 1 : 1 + decode;
}

namespace {

pa_status decode_append_impl(void *out, const void *q, const void *k_new, const void *v_new,
                             const int64_t *slot_mapping, void *k_cache, void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int max_context_len, int num_seqs,
                             int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, float scale, pa_dtype dtype, void *workspace,
                             size_t workspace_bytes, int partition_tokens, void *stream,
                             int window, bool early_start = false) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID;
  if (num_seqs == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_INVALID;
  const int group = num_q_heads / num_kv_heads;
  if ((window == 0 && uses_stream_kernel(group, block_size, num_blocks, num_kv_heads)) ||
      (window > 0 && window_on_stream(group, block_size, num_blocks, num_kv_heads))) {
    const FusedWrite fw{k_new, v_new, slot_mapping, k_cache, v_cache};
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                       max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim,
                       block_size, num_blocks, scale, dtype, workspace, workspace_bytes,
                       partition_tokens, stream, &fw, window, early_start);
  }
  // other shapes (and windows the partition kernel runs): the write kernel, then the decode
  const pa_status st = pa_reshape_and_cache(k_new, v_new, slot_mapping, num_seqs, k_cache,
                                            v_cache, num_blocks, num_kv_heads, block_size,
                                            head_dim, dtype, stream);
  if (st != PA_OK) return st;
  return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, scale, dtype, workspace, workspace_bytes, partition_tokens,
                     stream, nullptr, window);
}

}  // namespace

extern "C" pa_status pa_decode_append(void *out, const void *q, const void *k_new,
                                      const void *v_new, const int64_t *slot_mapping,
                                      void *k_cache, void *v_cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *context_lens,
                                      int max_context_len, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size,
                                      int num_blocks, float scale, pa_dtype dtype,
                                      void *workspace, size_t workspace_bytes,
                                      int partition_tokens, void *stream) {
  return decode_append_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                            max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                            dtype, workspace, workspace_bytes, partition_tokens, stream, 0);
}

extern "C" pa_status pa_decode_append_overlapped(
    void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slot_mapping,
    void *k_cache, void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, int max_context_len, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
    void *workspace, size_t workspace_bytes, int partition_tokens, void *stream) {
  return decode_append_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                            max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                            dtype, workspace, workspace_bytes, partition_tokens, stream, 0, true);
}

extern "C" pa_status pa_decode_append_window(
    void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slot_mapping,
    void *k_cache, void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, int max_context_len, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int window,
    pa_dtype dtype, void *workspace, size_t workspace_bytes, int partition_tokens, void *stream) {
  if (window <= 0) return PA_ERR_INVALID;
  return decode_append_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                            max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                            dtype, workspace, workspace_bytes, partition_tokens, stream, window);
}

extern "C" pa_status pa_decode_append_window_overlapped(
    void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slot_mapping,
    void *k_cache, void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, int max_context_len, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int window,
    pa_dtype dtype, void *workspace, size_t workspace_bytes, int partition_tokens, void *stream) {
  if (window <= 0) return PA_ERR_INVALID;
  return decode_append_impl(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                            max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                            num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                            dtype, workspace, workspace_bytes, partition_tokens, stream, window,
                            true);
}

bool pa_internal_pool_tensor_map(CUtensorMap *map, const void *base, long long rows, int head_dim,
                                 int box_rows, pa_dtype dtype) {
  return pool_tensor_map(map, base, rows, head_dim, box_rows, dtype);
}

size_t pa_internal_decode_need(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, int max_context_len,
                               int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
      block_size <= 0 || num_blocks <= 0 || (head_dim != 64 && head_dim != 128) ||
      max_context_len < 0 || partition_tokens < 0 || partition_tokens % kPartitionQuantum ||
      partition_tokens > kMaxPartitionTokens)
    return 0;
  return decode_need(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                     max_context_len, partition_tokens, 0);
}

pa_status pa_internal_decode_status(cudaStream_t stream, int32_t *code) {
  int value = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&value, g_decode_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_decode_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                              stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
  *code = value;
  return PA_OK;
}

extern "C" pa_status pa_device_status(void *stream, int32_t *code) {
  if (!code) return PA_ERR_INVALID;
  int32_t a = 0, b = 0, c = 0;
  pa_status st = pa_internal_cache_ops_status(static_cast<cudaStream_t>(stream), &a);
  if (st != PA_OK) return st;
  st = pa_internal_decode_status(static_cast<cudaStream_t>(stream), &b);
  if (st != PA_OK) return st;
  st = pa_internal_prefill_status(static_cast<cudaStream_t>(stream), &c);
  if (st != PA_OK) return st;
  *code = a | b | c;
  return PA_OK;
}
