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

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pa.h"
#include "pa_internal.h"

namespace {

__device__ int g_decode_error;

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 4;
constexpr int kTileBytes = 8192;                 // bytes of K (and of V) per stage
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// ------------------------------------------------------------------------------------ PTX wraps
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx_arrive(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` to complete, at most kWaitLimitNs; also give
// up when another thread of the CTA has raised *abort. Returns false on give-up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      atomicOr(&g_decode_error, PA_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// 1-D TMA bulk copy global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------------ element conversions
template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
  // 8 packed bf16 -> 8 floats (a bf16 is the upper half of a float)
  static __device__ __forceinline__ void to_f32(const uint4 &r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float a) {
    return __float2bfloat16_rn(a);
  }
  static __device__ __forceinline__ uint2 from_f32x4(float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b);
    __nv_bfloat162 hi = __floats2bfloat162_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
  }
};

template <>
struct Elem<__half> {
  static __device__ __forceinline__ void to_f32(const uint4 &r, float (&f)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
  static __device__ __forceinline__ __half from_f32(float a) { return __float2half_rn(a); }
  static __device__ __forceinline__ uint2 from_f32x4(float a, float b, float c, float d) {
    __half2 lo = __floats2half2_rn(a, b);
    __half2 hi = __floats2half2_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
  }
};

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
};

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
  const int nparts = len > 0 ? (len + p.partition_tokens - 1) / p.partition_tokens : 1;
  if (part >= nparts) return;
  const int t_begin = part * p.partition_tokens;
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
      for (int i = max(0, issued - kStages); i < issued; ++i) {
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
    const bool landed = mbar_wait_bounded(&full_bar[s], (i / kStages) & 1, abort_flag);
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

// ------------------------------------------------------------------------------ merge kernel
// One CTA per (q head, sequence), one thread per output element: combine the
// partitions' (max, sum, weighted V) states by log-sum-exp.
template <typename T, int D>
__global__ void __launch_bounds__(D) pa_decode_merge_kernel(
    void *out_, const float *__restrict__ ws_acc, const float *__restrict__ ws_ml,
    const int32_t *__restrict__ context_lens, int num_q_heads, int partition_tokens,
    int max_parts, int max_context_len, int cap) {
  const int hqi = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  int len = __ldg(context_lens + b);
  len = len < 0 ? 0 : min(min(len, cap), max_context_len);
  const int nparts = (len + partition_tokens - 1) / partition_tokens;
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

template <typename T, int D, int G>
pa_status launch_decode(const DecodeParams &prm, int num_seqs, void *out, cudaStream_t stream) {
  using L = Smem<T, D, G>;
  const size_t smem = L::bytes(prm.table_slice);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  static size_t configured[kMaxDevices] = {};  // largest dynamic smem set per device
  if (smem > configured[dev]) {
    if (cudaFuncSetAttribute(pa_decode_partition_kernel<T, D, G>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return PA_ERR_CUDA;
    configured[dev] = smem;
  }
  dim3 grid((unsigned)prm.max_parts, (unsigned)prm.num_kv_heads, (unsigned)num_seqs);
  pa_decode_partition_kernel<T, D, G><<<grid, kThreads, smem, stream>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (prm.max_parts > 1) {
    dim3 mgrid((unsigned)prm.num_q_heads, (unsigned)num_seqs);
    pa_decode_merge_kernel<T, D><<<mgrid, D, 0, stream>>>(
        out, prm.ws_acc, prm.ws_ml, prm.context_lens, prm.num_q_heads, prm.partition_tokens,
        prm.max_parts, prm.max_context_len, prm.max_blocks_per_seq * prm.block_size);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <typename T, int D>
pa_status dispatch_group(int group, const DecodeParams &prm, int num_seqs, void *out,
                         cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode<T, D, 1>(prm, num_seqs, out, stream);
    case 2: return launch_decode<T, D, 2>(prm, num_seqs, out, stream);
    case 4: return launch_decode<T, D, 4>(prm, num_seqs, out, stream);
    case 8: return launch_decode<T, D, 8>(prm, num_seqs, out, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <typename T>
pa_status dispatch_dim(int head_dim, int group, const DecodeParams &prm, int num_seqs, void *out,
                       cudaStream_t stream) {
  switch (head_dim) {
    case 64: return dispatch_group<T, 64>(group, prm, num_seqs, out, stream);
    case 128: return dispatch_group<T, 128>(group, prm, num_seqs, out, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

constexpr int kPartitionQuantum = 64;   // partitions are whole tiles for every head_dim
constexpr int kMaxPartitionTokens = 8192;
constexpr int kSmCount = 148;
constexpr int kCtasPerSm = 3;

int resolve_partition(int num_seqs, int num_kv_heads, int max_context_len, int requested) {
  if (requested > 0) return requested;
  return pa_decode_default_partition(num_seqs, num_kv_heads, max_context_len);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

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

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                           int head_dim, int max_context_len,
                                           int partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_context_len <= 0 || partition_tokens < 0)
    return 0;
  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  const long long parts = (max_context_len + pt - 1) / pt;
  if (parts <= 1) return 0;
  return (size_t)num_seqs * num_q_heads * parts * (head_dim + 2) * sizeof(float);
}

extern "C" pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, int max_context_len, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, float scale, pa_dtype dtype, void *workspace,
                               size_t workspace_bytes, int partition_tokens, void *stream) {
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

  const int pt = resolve_partition(num_seqs, num_kv_heads, max_context_len, partition_tokens);
  const int max_parts = max_context_len > 0 ? (max_context_len + pt - 1) / pt : 1;
  const size_t need =
      max_parts > 1 ? (size_t)num_seqs * num_q_heads * max_parts * (head_dim + 2) * sizeof(float)
                    : 0;
  if (need > workspace_bytes || (need && (!workspace || !aligned(workspace, 16))))
    return PA_ERR_INVALID;

  DecodeParams prm;
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.ws_acc = static_cast<float *>(workspace);
  prm.ws_ml = need ? static_cast<float *>(workspace) +
                         (size_t)num_seqs * num_q_heads * max_parts * head_dim
                   : nullptr;
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

  const int group = num_q_heads / num_kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PA_BF16) return dispatch_dim<__nv_bfloat16>(head_dim, group, prm, num_seqs, out, st);
  return dispatch_dim<__half>(head_dim, group, prm, num_seqs, out, st);
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
  int32_t a = 0, b = 0;
  pa_status st = pa_internal_cache_ops_status(static_cast<cudaStream_t>(stream), &a);
  if (st != PA_OK) return st;
  st = pa_internal_decode_status(static_cast<cudaStream_t>(stream), &b);
  if (st != PA_OK) return st;
  *code = a | b;
  return PA_OK;
}
