// pa_prefill.cu -- paged attention for several query tokens per sequence
// (prefill, or one chunk of a chunked prefill) on sm_100a.
//
// What it computes ("PagedAttention 核心思想解析", section 2.2: the rows of Q
// are cut into blocks, each block is scored against the sequence's K/V blocks
// found through the block table, and the partial results are merged by
// position): sequence b holds n = context_lens[b] positions; its
// m = q_start[b+1] - q_start[b] query tokens are its last m positions (their
// K/V already written to the pool), and the token at position p attends to
// positions [lo, p] -- lo = p + 1 - window under a sliding window, else 0.
//
// Two kernels compute it. The default (pa_prefill_tc_kernel, further down)
// runs both products on the 5th-generation tensor cores (tcgen05.mma, S, P
// and O in tensor memory, 256 query rows per CTA). The first version
// (pa_prefill_kernel, selected with -DPA_PREFILL_TCGEN05=0) uses mma.sync with
// register accumulators; its design:
//  * One CTA per (q head, 64 query tokens, sequence); the q heads of one kv
//    head are neighbours in the grid, so the CTAs sharing a K/V tile run
//    together and all but the first read it from L2. Tiles with the most keys
//    (the last query tiles of a sequence) are launched first.
//  * A producer warp streams the CTA's key tiles (64 keys) into a 2-stage ring
//    with 2-D TMA copies of each (block, kv head) piece (128-byte swizzle; the
//    same pool tensor maps as decode), guarded by full / empty mbarriers.
//  * Four consumer warps own 16 query rows each. Per tile: S = Q K^T with
//    mma.sync m16n8k16 (Q fragments stay in registers for the whole loop, K
//    from ldmatrix on the swizzled panels), the causal / window mask on the
//    tiles that need it, online softmax in the log2 domain, and O += P V with
//    P rebuilt in registers as A fragments and V from ldmatrix.trans. The
//    running sum uses the rounded weights, so the result is an exact weighted
//    average of V. Rows of V past the sequence's last position (never written,
//    may hold anything) are zeroed in shared memory before the product.
//  * Every wait is bounded; block ids and lengths are range-checked and a bad
//    one is skipped and reported in the device error word, never accessed.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "pa.h"
#include "pa_internal.h"
#include "pa_ptx.cuh"

// Which kernel pa_prefill runs: 1 = tcgen05 (tensor memory accumulators), 0 =
// mma.sync (register accumulators).
#ifndef PA_PREFILL_TCGEN05
#define PA_PREFILL_TCGEN05 1
#endif

namespace {

__device__ int g_prefill_error;

constexpr int kQTile = 64;       // query tokens per CTA
constexpr int kWarps = 4;        // consumer warps, 16 query rows each
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kStages = 2;
constexpr int kPanelBytes = 64 * 128;  // 64 rows x 64 columns of 2 bytes, 128-byte swizzled
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

struct PrefillParams {
  void *out;                  // [T][Hq][D]
  const void *q;              // [T][Hq][D]
  const int32_t *block_tables;
  const int32_t *context_lens;
  const int32_t *q_start;     // [B + 1]
  int max_blocks_per_seq;
  int max_context_len;
  int num_tokens;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int window;
  int q_tiles;                // grid.y (tcgen05 kernel: query tiles of an item)
  float scale_log2;
  int pair_heads;             // tcgen05 kernel: 1 = an item is two q heads of one kv head
  const int *order;           // tcgen05 kernel: (sequence, query tile) pairs in the order
                              // items take them, or null for index order
};

template <int D>
struct Layout {
  static constexpr int kPanels = D / 64;
  static constexpr int kQBytes = kPanels * kPanelBytes;          // 64 query rows
  static constexpr int kStageBytes = 2 * kPanels * kPanelBytes;  // K panels, then V panels
  static constexpr int kRingOffset = kQBytes;
  static constexpr int kBarOffset = kRingOffset + kStages * kStageBytes;
  static constexpr int kFlagOffset = kBarOffset + 2 * kStages * 8;
  static constexpr int kBytes = 1024 + kFlagOffset + 16;  // + slack to align to 1 KB
};

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      atomicOr(&g_prefill_error, PA_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz, one
// instruction; its error is far below the rounding of the 16-bit weights it
// feeds, and -inf gives 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// First position the token at position p attends to.
__device__ __forceinline__ int first_key(int p, int window) {
  return window > 0 && p + 1 > window ? p + 1 - window : 0;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) pa_prefill_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const PrefillParams p) {
  using L = Layout<D>;
  constexpr int kKTile = 64;      // keys per stage
  constexpr int KSTEPS = D / 16;  // k-steps of Q K^T
  constexpr int NT_O = D / 8;     // n-tiles of the output row block

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
  uint64_t *empty_bar = full_bar + kStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kFlagOffset);
  const uint32_t qsm = smem_u32(smem);
  const uint32_t ring = smem_u32(smem + L::kRingOffset);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int qt = p.q_tiles - 1 - (int)blockIdx.y;  // the longest tiles first
  const int b = blockIdx.z;
  const int G = p.num_q_heads / p.num_kv_heads;
  const int kvh = h / G;
  const int bs = p.block_size;
  const int cap = p.max_blocks_per_seq * bs;

  // ---- this CTA's query rows and key range (the same in every thread)
  int n = __ldg(p.context_lens + b);
  const int qs0 = __ldg(p.q_start + b), qs1 = __ldg(p.q_start + b + 1);
  int m = qs1 - qs0;
  bool bad = false;
  if (n < 0 || n > cap || n > p.max_context_len) {
    bad = true;
    n = n < 0 ? 0 : min(min(n, cap), p.max_context_len);
  }
  if (m < 0 || m > n || qs0 < 0 || qs1 > p.num_tokens) {
    bad = true;
    m = 0;
  }
  if (bad && tid == 0 && h == 0 && blockIdx.y == 0)
    atomicOr(&g_prefill_error, PA_DEVERR_CONTEXT_LEN);
  const int q0 = qt * kQTile;
  if (q0 >= m) return;  // no query rows here (uniform)
  const int rows = min(kQTile, m - q0);
  const int p_first = n - m + q0;       // position of the first query row
  const int p_last = p_first + rows - 1;
  const int align = bs < kKTile ? bs : kKTile;
  const int k_base = first_key(p_first, p.window) & ~(align - 1);  // block / 64-key aligned
  const int ntiles = (p_last + 1 - k_base + kKTile - 1) / kKTile;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kWarps) {
    // ======================================================================== producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)));
    }
    const int32_t *row = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    const int box_rows = align;
    const uint32_t box_bytes = 2u * L::kPanels * box_rows * 128u;  // K and V
    int issued = 0;
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % kStages;
      if (i >= kStages && !wait_bounded(&empty_bar[s], ((i / kStages) & 1) ^ 1, abort_flag))
        break;
      __syncwarp();
      const int t0 = k_base + i * kKTile;
      const int t_end = min(t0 + kKTile, n);  // keys past n are never read
      // boxes of this tile: whole blocks (block_size <= 64) or one 64-key slice
      const int nbox = t_end > t0 ? (bs <= kKTile ? (t_end - 1) / bs - t0 / bs + 1 : 1) : 0;
      int phys = -1;
      bool ok = false;
      if (lane < nbox) {
        const int lb = t0 / bs + lane;
        phys = lb < p.max_blocks_per_seq ? __ldg(row + lb) : -1;
        ok = phys >= 0 && phys < p.num_blocks;
        if (!ok) atomicOr(&g_prefill_error, PA_DEVERR_BLOCK_ID);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_expect_tx_arrive(&full_bar[s], __popc(okmask) * box_bytes);
      __syncwarp();
      // one lane per (box, operand, panel): lane = box * 2 * kPanels + which * kPanels + pn
      const int per_box = 2 * L::kPanels;
      const int box = lane / per_box;
      const int which = (lane / L::kPanels) % 2;
      const int pn = lane % L::kPanels;
      const int box_phys = __shfl_sync(0xffffffffu, phys, box & 31);
      if (box < nbox && ((okmask >> box) & 1u)) {
        const int r0 = bs > kKTile ? t0 % bs : 0;
        const int srow = bs > kKTile ? 0 : box * bs;
        const int y = (box_phys * p.num_kv_heads + kvh) * bs + r0;
        tma_load_2d(ring + s * L::kStageBytes + (which * L::kPanels + pn) * kPanelBytes + srow * 128,
                    which ? &tmap_v : &tmap_k, pn * 64, y, &full_bar[s]);
      }
      issued = i + 1;
    }
    // do not leave while copies may still land in this CTA's shared memory
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i) {
        const int s = i % kStages;
        const unsigned long long t_start = global_ns();
        while (!mbar_try_wait(&full_bar[s], (i / kStages) & 1)) {
          if (global_ns() - t_start > kWaitLimitNs) {
            atomicOr(&g_prefill_error, PA_DEVERR_TIMEOUT);
            break;
          }
        }
      }
    }
    return;
  }

  // ========================================================================== consumers
  const int g = lane >> 2, t = lane & 3;
  const int wrow = warp * 16;
  // positions of this thread's two query rows (rows past the chunk are clamped
  // to the last position: computed, never stored)
  const int pr0 = min(p_first + wrow + g, n - 1);
  const int pr1 = min(p_first + wrow + g + 8, n - 1);
  const int lo0 = first_key(pr0, p.window), lo1 = first_key(pr1, p.window);
  const int p_warp_first = p_first + wrow;
  const int p_warp_last = min(p_first + wrow + 15, n - 1);

  // ---- Q rows of this warp -> swizzled shared memory -> A fragments (kept)
  {
    const T *qg = static_cast<const T *>(p.q);
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int c = lane; c < 16 * kChunks; c += 32) {
      const int r = c / kChunks, ch = c % kChunks;
      const int qrow = wrow + r;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (qrow < rows)
        v = __ldg(reinterpret_cast<const uint4 *>(
                      qg + ((size_t)(qs0 + q0 + qrow) * p.num_q_heads + h) * D) + ch);
      *reinterpret_cast<uint4 *>(smem + (ch / 8) * kPanelBytes + qrow * 128 +
                                 (((ch % 8) ^ (qrow & 7)) << 4)) = v;
    }
    __syncwarp();
  }
  uint32_t qa[KSTEPS][4];
  {
    const int r = wrow + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk)
      ldsm_x4(swz(qsm + (kk / 4) * kPanelBytes, r, 2 * (kk % 4) + (lane >> 4)), qa[kk]);
  }

  float o[NT_O][4];
#pragma unroll
  for (int x = 0; x < NT_O; ++x) o[x][0] = o[x][1] = o[x][2] = o[x][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int kb_row = (lane & 7) + 8 * (lane >> 4);         // K ldmatrix: key row in 16
  const int kb_chk = (lane >> 3) & 1;                      //             d chunk in pair
  const int vb_row = (lane & 7) + 8 * ((lane >> 3) & 1);   // V ldmatrix.trans: key row
  const int vb_chk = lane >> 4;                            //                   d chunk

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    const bool landed = wait_bounded(&full_bar[s], (i / kStages) & 1, abort_flag);
    __syncwarp();
    const int t0 = k_base + i * kKTile;
    const uint32_t kst = ring + s * L::kStageBytes;
    const uint32_t vst = kst + L::kPanels * kPanelBytes;
    // rows of V outside every row's keys -- past the sequence's end (never
    // loaded, or unwritten slots) or before the first row's window (released
    // slots) -- may hold anything: zero them before any warp multiplies by them
    const int nvalid = min(kKTile, n - t0);
    const int nskip = max(0, first_key(p_first, p.window) - t0);
    if (nvalid < kKTile || nskip > 0) {
      unsigned char *vz = smem + L::kRingOffset + s * L::kStageBytes + L::kPanels * kPanelBytes;
      for (int r = warp * 4 + (lane >> 3); r < kKTile; r += 16) {
        if (r >= nskip && r < nvalid) continue;
#pragma unroll
        for (int pn = 0; pn < L::kPanels; ++pn)
          *reinterpret_cast<uint4 *>(vz + pn * kPanelBytes + r * 128 + (lane & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
    }
    // a warp whose rows all precede this tile, or whose windows all start after
    // it, has nothing to add
    if (landed && t0 <= p_warp_last && t0 + kKTile > first_key(p_warp_first, p.window)) {
      // ---- S = Q K^T: 16 rows x 64 keys (8 n-tiles of 8 keys)
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {  // pairs of n-tiles
          uint32_t kb[4];
          ldsm_x4(swz(kst + (kk / 4) * kPanelBytes, np * 16 + kb_row, 2 * (kk % 4) + kb_chk), kb);
          Mma<T>::run(sc[2 * np], qa[kk], kb[0], kb[1]);
          Mma<T>::run(sc[2 * np + 1], qa[kk], kb[2], kb[3]);
        }
      }
      // ---- scale, mask, online softmax (log2 domain)
      const bool need_mask = t0 + kKTile - 1 > p_warp_first ||
                             (p.window > 0 && t0 < first_key(p_warp_last, p.window));
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kp = t0 + nt * 8 + 2 * t + e;
          float a = sc[nt][e] * p.scale_log2, c = sc[nt][2 + e] * p.scale_log2;
          if (need_mask) {
            a = (kp <= pr0 && kp >= lo0) ? a : -INFINITY;
            c = (kp <= pr1 && kp >= lo1) ? c : -INFINITY;
          }
          sc[nt][e] = a;
          sc[nt][2 + e] = c;
          mx0 = fmaxf(mx0, a);
          mx1 = fmaxf(mx1, c);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = m0 == -INFINITY ? 0.f : exp2f(m0 - b0);
      const float al1 = m1 == -INFINITY ? 0.f : exp2f(m1 - b1);
      m0 = mn0;
      m1 = mn1;
      // P as A fragments of the 4 k-steps of P V (keys 16kk .. 16kk + 15)
      uint32_t pa[4][4];
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int nt = 2 * kk + half;
          float r00, r01, r10, r11;
          pa[kk][half * 2] = Mma<T>::pack(exp2f(sc[nt][0] - b0), exp2f(sc[nt][1] - b0), r00, r01);
          pa[kk][half * 2 + 1] =
              Mma<T>::pack(exp2f(sc[nt][2] - b1), exp2f(sc[nt][3] - b1), r10, r11);
          rs0 += r00 + r01;
          rs1 += r10 + r11;
        }
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int x = 0; x < NT_O; ++x) {
        o[x][0] *= al0;
        o[x][1] *= al0;
        o[x][2] *= al1;
        o[x][3] *= al1;
      }
      // ---- O += P V: for each pair of 8-wide d n-tiles, 4 k-steps of 16 keys
#pragma unroll
      for (int x = 0; x < NT_O / 2; ++x) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t vb[4];
          ldsm_x4_trans(swz(vst + (x / 4) * kPanelBytes, kk * 16 + vb_row, 2 * (x % 4) + vb_chk), vb);
          Mma<T>::run(o[2 * x], pa[kk], vb[0], vb[1]);
          Mma<T>::run(o[2 * x + 1], pa[kk], vb[2], vb[3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }

  // ---- normalise, stage the warp's rows in shared memory, store them
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  // the Q staging rows of this warp are free again (its fragments are in registers)
#pragma unroll
  for (int x = 0; x < NT_O; ++x) {
    const int col = x * 8 + 2 * t;  // element column; chunk col / 8, offset (col % 8) * 2
    float r;
    const uint32_t w0 = Mma<T>::pack(o[x][0] * inv0, o[x][1] * inv0, r, r);
    const uint32_t w1 = Mma<T>::pack(o[x][2] * inv1, o[x][3] * inv1, r, r);
    const int r0 = wrow + g, r1 = wrow + g + 8;
    *reinterpret_cast<uint32_t *>(smem + (col / 64) * kPanelBytes + r0 * 128 +
                                  ((((col % 64) / 8) ^ (r0 & 7)) << 4) + (col % 8) * 2) = w0;
    *reinterpret_cast<uint32_t *>(smem + (col / 64) * kPanelBytes + r1 * 128 +
                                  ((((col % 64) / 8) ^ (r1 & 7)) << 4) + (col % 8) * 2) = w1;
  }
  __syncwarp();
  {
    T *og = static_cast<T *>(p.out);
    constexpr int kChunks = D / 8;
    for (int c = lane; c < 16 * kChunks; c += 32) {
      const int r = c / kChunks, ch = c % kChunks;
      const int qrow = wrow + r;
      if (qrow >= rows) continue;
      const uint4 v = *reinterpret_cast<const uint4 *>(smem + (ch / 8) * kPanelBytes + qrow * 128 +
                                                       (((ch % 8) ^ (qrow & 7)) << 4));
      *(reinterpret_cast<uint4 *>(og + ((size_t)(qs0 + q0 + qrow) * p.num_q_heads + h) * D) + ch) = v;
    }
  }
}

// ============================================================ tcgen05 kernel (5th-gen tensor cores)
// Same computation on tcgen05.mma, with every operand of P V but V in tensor
// memory, as a persistent kernel: one CTA per SM takes work items one after another
// from a counter (in the order prefill_order_kernel wrote: the items reading the most
// key tiles first), and fetches the next item's Q and K/V tiles while the current one
// computes, so neither a CTA launch nor the first fetches of an item leave the SM
// idle. An item is two groups of 128 query rows (one tcgen05 M each) that read the
// same keys: with an even number of q heads per kv head, the same 128 query tokens
// of two q heads of one kv head (the groups then need the same tiles); otherwise
// 256 query tokens of one q head, split in two (the second group then needs one
// tile more). The groups share every K/V tile of 128 keys and take turns on the
// tensor core, so one group's softmax overlaps the other group's products.
//   warp 0      takes items, publishes each item's extent, stages its Q rows (TMA,
//               once the previous item's last S has read the Q buffer) and its
//               128-key K and V tiles (TMA) into two rings (3 K slots and 2 V slots
//               at head_dim 128; 6 and 4 at 64);
//   warp 1      allocates TMEM (512 columns: per group one S/P buffer of 128
//               columns and O); its lane 0 issues, item after item, per group: O +=
//               P V with P read from TMEM once the group's softmax wrote P and V
//               landed (the item's first one once the previous item's O was read
//               out), then at once the group's next S = Q K^T (M = 128, N = 128: the
//               shape the tensor core runs at its full rate), committing each to an
//               mbarrier; a K slot goes back once both groups' S read it, a V slot
//               once both groups' P V did;
//   warps 2-9   one thread per query row (group = (warp - 2) / 4, TMEM lane =
//               32 * (warp % 4) + lane): per tile read its S row from TMEM, mask,
//               online softmax in the log2 domain, and write its P row (16-bit, two
//               per column) over the first half of the S row it came from; at the
//               end of an item O / l goes from TMEM to global memory. The tensor
//               core runs its operations in issue order, so the next S cannot
//               overwrite P before the P V that reads it.
//               O is rescaled in TMEM only when the row max grows by more than
//               2^8 (the weights against the stale max stay <= 2^8 and the final
//               division by the matching sum keeps the result exact); l sums the
//               same rounded weights the product uses.
namespace t5 {

constexpr int kM = 128;        // query rows per group (tcgen05 M)
constexpr int kGroups = 2;
constexpr int kN = 128;        // keys per tile (tcgen05 N of S, K of P V)
constexpr int kThreads = (2 + 4 * kGroups) * 32;
// group g: S/P buffer at 256g (P in its first 64 columns), O at 256g + 128
constexpr uint32_t kTmemCols = 512;
constexpr float kLazyRescale = 8.f;  // log2 of the growth that forces an O rescale

// One work item as the producer publishes it to the other warps.
struct Item {
  int valid;        // 0: no more items
  int h, b;         // q head (of group 0), sequence
  int qs0, q0;      // first query row of the sequence in q / out, first row of the item in it
  int rows;         // query rows of the item (<= 128 with two heads, else <= 256)
  int n;            // positions of the sequence
  int p_first;      // position of the item's first query row
  int k_base;       // first key of the item's first tile
  int gtiles[kGroups];  // tiles each group needs
  int ntiles;       // tiles of the item (the larger of the two)
};

template <int D>
struct Lay {
  static constexpr int kPanels = D / 64;
  // Separate K and V rings: a K slot is free again once both groups' S have read
  // it, long before the tile's P V, so K tiles are fetched further ahead. At
  // head_dim 128: 64 KB of Q + 3 K slots + 2 V slots of 32 KB (224 KB); at 64:
  // 32 KB of Q + 6 + 4 slots of 16 KB.
  static constexpr int kKStages = D == 128 ? 3 : 6;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr int kQPanel = kGroups * kM * 128;          // 256 rows x 128 bytes
  static constexpr int kQBytes = kPanels * kQPanel;
  static constexpr int kKVPanel = kN * 128;                   // 128 rows x 128 bytes
  static constexpr int kSlotBytes = kPanels * kKVPanel;       // one operand of one tile
  static constexpr int kKRingOff = kQBytes;
  static constexpr int kVRingOff = kKRingOff + kKStages * kSlotBytes;
  static constexpr int kBarOff = kVRingOff + kVStages * kSlotBytes;
  // k_full[K] k_empty[K] v_full[V] v_empty[V] q_full q_free item_full[2]
  // item_free[2] mma_done, then per group s_full p_full pv_done o_free
  static constexpr int kNumBars = 2 * kKStages + 2 * kVStages + 7 + 4 * kGroups;
  static constexpr int kItemOff = kBarOff + kNumBars * 8;
  static constexpr int kTmemOff = kItemOff + 2 * (int)sizeof(Item);
  static constexpr int kFlagOff = kTmemOff + 8;
  static constexpr int kBytes = 1024 + kFlagOff + 16;
  static_assert(kBytes <= 227 * 1024, "shared memory of one CTA");
};

}  // namespace t5

template <typename T, int D>
__global__ void __launch_bounds__(t5::kThreads, 1) pa_prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const __grid_constant__ CUtensorMap tmap_q, const PrefillParams p, unsigned *work) {
  using L = t5::Lay<D>;
  using t5::Item;
  constexpr int kM = t5::kM, kN = t5::kN, NK = L::kKStages, NV = L::kVStages, NG = t5::kGroups;
  constexpr uint32_t kFmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t kIdescS = umma_idesc_f16(kFmt, 0, 0, kN, kM);  // Q (K-major) . K (K-major)
  constexpr uint32_t kIdescO = umma_idesc_f16(kFmt, 0, 1, D, kM);   // P (TMEM) . V (MN-major)

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint64_t *k_full = bars, *k_empty = bars + NK, *v_full = bars + 2 * NK;
  uint64_t *v_empty = v_full + NV, *q_full = v_full + 2 * NV, *q_free = q_full + 1;
  uint64_t *item_full = q_free + 1, *item_free = item_full + 2, *mma_done = item_free + 2;
  // per group g: s_full, p_full, pv_done (each completes once per tile of the group),
  // o_free (once per item: the group's O has been read out)
  auto s_full = [&](int g) { return mma_done + 1 + g * 4; };
  auto p_full = [&](int g) { return mma_done + 1 + g * 4 + 1; };
  auto pv_done = [&](int g) { return mma_done + 1 + g * 4 + 2; };
  auto o_free = [&](int g) { return mma_done + 1 + g * 4 + 3; };
  Item *items = reinterpret_cast<Item *>(smem + L::kItemOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kFlagOff);
  const uint32_t q_sm = smem_u32(smem);
  const uint32_t k_ring = smem_u32(smem + L::kKRingOff);
  const uint32_t v_ring = smem_u32(smem + L::kVRingOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bs = p.block_size;
  const int cap = p.max_blocks_per_seq * bs;
  const int align = bs < kN ? bs : kN;
  const int G = p.num_q_heads / p.num_kv_heads;
  const bool pair = p.pair_heads != 0;
  const int h_items = pair ? p.num_q_heads / 2 : p.num_q_heads;  // items per query tile
  // group g of an item: q head h + g * g_head, query rows from q0 + g * g_row
  const int g_head = pair ? 1 : 0, g_row = pair ? 0 : kM;
  const long long n_items = (long long)h_items * p.q_tiles * p.num_seqs;

  if (tid == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);  // one tcgen05.commit per use
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_free[i], 1 + 4 * NG);  // the issuing thread and every softmax warp
    }
    mbar_init(mma_done, 1);
    for (int g = 0; g < NG; ++g) {
      mbar_init(s_full(g), 1);
      mbar_init(p_full(g), 128);
      mbar_init(pv_done(g), 1);
      mbar_init(o_free(g), 128);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, t5::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ======================================================================== producer
    // Launched as a programmatic dependent of prefill_order_kernel, the CTA may have
    // started before that kernel finished: wait for it before the first read of the
    // item order or the work counter (a no-op otherwise). Nothing else the kernel
    // reads is written by it.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)));
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)));
    }
    const uint32_t box_bytes = (uint32_t)L::kPanels * align * 128u;  // one operand of one box
    long long kt = 0, vt = 0;  // K / V tiles loaded so far (over all items)
    int nq = 0;                // items whose Q rows were loaded (those with tiles)
    for (int it = 0;; ++it) {
      // ---- the next work item: q head (or head pair) fastest, then the (sequence,
      // query tile) pairs in the given order
      long long k = 0;
      if (lane == 0) k = atomicAdd(work, 1u);
      k = __shfl_sync(0xffffffffu, k, 0);
      Item I;
      I.valid = k < n_items;
      if (I.valid) {
        const int hi = (int)(k % h_items);
        I.h = pair ? 2 * hi : hi;
        const long long u = k / h_items;  // (sequence, query tile) pair of the item
        const int pu = p.order ? __ldg(p.order + u) : (int)u;
        const int qt = p.q_tiles - 1 - pu % p.q_tiles;
        I.b = pu / p.q_tiles;
        int n = __ldg(p.context_lens + I.b);
        const int qs0 = __ldg(p.q_start + I.b), qs1 = __ldg(p.q_start + I.b + 1);
        int m = qs1 - qs0;
        bool bad = false;
        if (n < 0 || n > cap || n > p.max_context_len) {
          bad = true;
          n = n < 0 ? 0 : min(min(n, cap), p.max_context_len);
        }
        if (m < 0 || m > n || qs0 < 0 || qs1 > p.num_tokens) {
          bad = true;
          m = 0;
        }
        if (bad && lane == 0 && I.h == 0 && qt == p.q_tiles - 1)
          atomicOr(&g_prefill_error, PA_DEVERR_CONTEXT_LEN);
        I.n = n;
        I.qs0 = qs0;
        const int item_rows = pair ? kM : NG * kM;
        I.q0 = qt * item_rows;
        I.rows = m > I.q0 ? min(item_rows, m - I.q0) : 0;
        I.p_first = n - m + I.q0;
        I.k_base = first_key(I.p_first, p.window) & ~(align - 1);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          const int grows = min(kM, I.rows - g * g_row);
          I.gtiles[g] =
              grows > 0 ? (I.p_first + g * g_row + grows - 1 + 1 - I.k_base + kN - 1) / kN : 0;
        }
        I.ntiles = max(I.gtiles[0], I.gtiles[1]);
      }
      // publish it (the slot's previous item has been read by every other warp)
      const int slot = it & 1;
      if (it >= 2) wait_bounded(&item_free[slot], ((it >> 1) - 1) & 1, abort_flag);
      if (lane == 0) {
        items[slot] = I;
        mbar_arrive(&item_full[slot]);
      }
      __syncwarp();
      if (!I.valid) break;
      if (I.ntiles == 0) continue;  // no query rows in this tile of the sequence
      // ---- its Q rows, once the previous item's last S has read the buffer
      if (nq > 0 && !wait_bounded(q_free, (nq - 1) & 1, abort_flag)) break;
      if (lane == 0) {
        mbar_expect_tx_arrive(q_full, (uint32_t)L::kQBytes);
        for (int pn = 0; pn < L::kPanels; ++pn)
#pragma unroll
          for (int g = 0; g < NG; ++g)
            tma_load_3d(q_sm + pn * L::kQPanel + g * kM * 128, &tmap_q, pn * 64,
                        I.h + g * g_head, I.qs0 + I.q0 + g * g_row, q_full);
      }
      __syncwarp();
      ++nq;
      // ---- its K and V tiles
      const int32_t *row = p.block_tables + (size_t)I.b * p.max_blocks_per_seq;
      const int kvh = I.h / G;
      auto load = [&](int i, int which, long long gi) {
        const int t0 = I.k_base + i * kN;
        const int t_end = min(t0 + kN, I.n);
        const int nbox = t_end > t0 ? (bs <= kN ? (t_end - 1) / bs - t0 / bs + 1 : 1) : 0;
        int phys = -1;
        bool ok = false;
        if (lane < nbox) {
          const int lb = t0 / bs + lane;
          phys = lb < p.max_blocks_per_seq ? __ldg(row + lb) : -1;
          ok = phys >= 0 && phys < p.num_blocks;
          if (!ok && which == 0) atomicOr(&g_prefill_error, PA_DEVERR_BLOCK_ID);
        }
        const unsigned okmask = __ballot_sync(0xffffffffu, ok);
        uint64_t *bar = which ? &v_full[gi % NV] : &k_full[gi % NK];
        if (lane == 0) mbar_expect_tx_arrive(bar, __popc(okmask) * box_bytes);
        __syncwarp();
        const uint32_t slot_addr = which ? v_ring + (uint32_t)(gi % NV) * L::kSlotBytes
                                         : k_ring + (uint32_t)(gi % NK) * L::kSlotBytes;
        for (int c0 = 0; c0 < nbox * L::kPanels; c0 += 32) {
          const int c = c0 + lane;
          const int box = c / L::kPanels;
          const int box_phys = __shfl_sync(0xffffffffu, phys, box & 31);
          if (c < nbox * L::kPanels && ((okmask >> box) & 1u)) {
            const int pn = c % L::kPanels;
            const int r0 = bs > kN ? t0 % bs : 0;
            const int srow = bs > kN ? 0 : box * bs;
            const int y = (box_phys * p.num_kv_heads + kvh) * bs + r0;
            tma_load_2d(slot_addr + pn * L::kKVPanel + srow * 128, which ? &tmap_v : &tmap_k,
                        pn * 64, y, bar);
          }
        }
      };
      // K tiles first (S needs them first) and as far ahead as the K ring allows;
      // a V tile once its K tile is out and a V slot is free
      int ik = 0, iv = 0;
      unsigned long long idle_since = global_ns();
      bool stop = false;
      while (ik < I.ntiles || iv < I.ntiles) {
        bool progress = false;
        if (ik < I.ntiles && (kt < NK || mbar_try_wait(&k_empty[kt % NK], ((kt / NK) & 1) ^ 1))) {
          load(ik++, 0, kt++);
          progress = true;
        }
        if (iv < ik && (vt < NV || mbar_try_wait(&v_empty[vt % NV], ((vt / NV) & 1) ^ 1))) {
          load(iv++, 1, vt++);
          progress = true;
        }
        if (progress) {
          idle_since = global_ns();
        } else if (*abort_flag || global_ns() - idle_since > kWaitLimitNs) {
          if (lane == 0 && !*abort_flag) atomicOr(&g_prefill_error, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          stop = true;
          break;
        }
      }
      if (stop) break;
    }
    // after a give-up, let the copies already issued land (bounded) before the CTA
    // exits: the last copy into each K / V slot and the last Q copy
    if (*abort_flag && lane == 0) {
      const unsigned long long t_start = global_ns();
      auto settle = [&](uint64_t *bar, uint32_t parity) {
        while (!mbar_try_wait(bar, parity) && global_ns() - t_start < kWaitLimitNs) {
        }
      };
      for (long long i = kt > NK ? kt - NK : 0; i < kt; ++i) settle(&k_full[i % NK], (i / NK) & 1);
      for (long long i = vt > NV ? vt - NV : 0; i < vt; ++i) settle(&v_full[i % NV], (i / NV) & 1);
      if (nq > 0) settle(q_full, (nq - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ====================================================================== MMA issuer
    if (lane == 0) {
      long long ts[NG], tp[NG];  // S / P V issued so far per group (over all items)
      long long krel = 0, vrel = 0;  // K / V tiles released so far
      long long kb = 0;              // K (and V) tiles of the items before this one
#pragma unroll
      for (int g = 0; g < NG; ++g) ts[g] = tp[g] = 0;
      int nq = 0;  // items whose Q was loaded (those with tiles)
      bool go = true;
      for (int it = 0; go; ++it) {
        const int slot = it & 1;
        if (!wait_bounded(&item_full[slot], (it >> 1) & 1, abort_flag)) break;
        const Item I = items[slot];
        mbar_arrive(&item_free[slot]);
        if (!I.valid) break;
        if (I.ntiles == 0) continue;
        if (!wait_bounded(q_full, nq & 1, abort_flag)) break;
        tc_fence_after();
        int ns[NG], npv[NG];
#pragma unroll
        for (int g = 0; g < NG; ++g) ns[g] = npv[g] = 0;
        int released_k = 0, released_v = 0;
        bool q_released = false;
        unsigned long long idle_since = global_ns();
        while (true) {
          bool done = true, progress = false;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            if (npv[g] < I.gtiles[g]) done = false;
            // this group's P V first (the item's first one once the group's O of the
            // previous item was read out), then at once its next S
            const int jp = npv[g];
            const long long gv = kb + jp;  // global V tile
            if (jp < ns[g] && mbar_try_wait(p_full(g), tp[g] & 1) &&
                mbar_try_wait(&v_full[gv % NV], (gv / NV) & 1) &&
                (jp > 0 || nq == 0 || mbar_try_wait(o_free(g), (nq - 1) & 1))) {
              tc_fence_after();
              const uint32_t vaddr = v_ring + (uint32_t)(gv % NV) * L::kSlotBytes;
#pragma unroll
              for (int kk = 0; kk < kN / 16; ++kk)
                umma_f16_ts(tmem + g * 256 + 128, tmem + g * 256 + kk * 8,
                            umma_desc_sw128(vaddr + kk * 16 * 128, L::kKVPanel, 1024),
                            kIdescO, jp > 0 || kk > 0);
              umma_commit(pv_done(g));
              ++npv[g];
              ++tp[g];
              progress = true;
            }
            const int js = ns[g];
            const long long gk = kb + js;  // global K tile
            if (js < I.gtiles[g] && npv[g] >= js &&
                mbar_try_wait(&k_full[gk % NK], (gk / NK) & 1)) {
              tc_fence_after();
              const uint32_t kaddr = k_ring + (uint32_t)(gk % NK) * L::kSlotBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                umma_f16(tmem + g * 256,
                         umma_desc_sw128(q_sm + (kk / 4) * L::kQPanel + g * kM * 128 +
                                             (kk % 4) * 32,
                                         16, 1024),
                         umma_desc_sw128(kaddr + (kk / 4) * L::kKVPanel + (kk % 4) * 32, 16, 1024),
                         kIdescS, kk > 0);
              umma_commit(s_full(g));
              ++ns[g];
              ++ts[g];
              progress = true;
            }
          }
          // once every S of the item is out, the Q buffer goes back to the producer
          if (!q_released && ns[0] == I.gtiles[0] && ns[1] == I.gtiles[1]) {
            umma_commit(q_free);
            q_released = true;
          }
          // release, in order, every K tile all of whose readers have issued S, and
          // every V tile all of whose readers have issued P V (each commit arrives
          // once the products issued before it have finished reading)
          while (released_k < I.ntiles) {
            bool all = true;
#pragma unroll
            for (int g = 0; g < NG; ++g)
              if (released_k < I.gtiles[g] && ns[g] <= released_k) all = false;
            if (!all) break;
            umma_commit(&k_empty[krel % NK]);
            ++krel;
            ++released_k;
          }
          while (released_v < I.ntiles) {
            bool all = true;
#pragma unroll
            for (int g = 0; g < NG; ++g)
              if (released_v < I.gtiles[g] && npv[g] <= released_v) all = false;
            if (!all) break;
            umma_commit(&v_empty[vrel % NV]);
            ++vrel;
            ++released_v;
          }
          if (done && released_v == I.ntiles) break;
          const unsigned long long now = global_ns();
          if (progress) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs || *abort_flag) {
            *abort_flag = 1;
            atomicOr(&g_prefill_error, PA_DEVERR_TIMEOUT);
            go = false;
            break;
          }
        }
        kb += I.ntiles;
        ++nq;
      }
      // every product issued so far has finished before TMEM is released
      umma_commit(mma_done);
      wait_bounded(mma_done, 0, abort_flag);
    }
    __syncwarp();
  } else {
    // ====================================================== softmax, one row per thread
    const int grp = (warp - 2) / 4;
    const int r = 32 * (warp % 4) + lane;          // row in the group == TMEM lane
    const int R = grp * g_row + r;                 // row in the item
    const uint32_t trow = tmem + ((uint32_t)(32 * (warp % 4)) << 16) + grp * 256;
    long long tg = 0;   // tiles of this group so far (over all items)
    long long vg = 0;   // V tiles of the items before this one
    for (int it = 0;; ++it) {
      const int slot = it & 1;
      if (!wait_bounded(&item_full[slot], (it >> 1) & 1, abort_flag)) break;
      const Item I = items[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_free[slot]);
      if (!I.valid) break;
      if (I.ntiles == 0) continue;
      const int my_tiles = I.gtiles[grp];
      const int rows = I.rows, n = I.n, k_base = I.k_base, p_first = I.p_first;
      const int pr = min(p_first + R, n - 1);       // rows past the chunk: computed, not stored
      const int lo = first_key(pr, p.window);
      const int lo_first = first_key(p_first, p.window);
      const int wr0 = min(p_first + grp * g_row + 32 * (warp % 4), n - 1);
      const int wr1 = min(p_first + grp * g_row + 32 * (warp % 4) + 31, n - 1);
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < my_tiles; ++j) {
        const long long t = tg + j;
        const int t0 = k_base + j * kN;
        wait_bounded(s_full(grp), t & 1, abort_flag);
        tc_fence_after();
        uint32_t sv[kN];
#pragma unroll
        for (int c4 = 0; c4 < kN / 32; ++c4)
          tmem_ld32(trow + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c4 * 32]));
        tmem_wait_ld();
        // max of the raw scores (the scale is positive); masked keys become -inf.
        // The mask only matters on tiles that reach past a row of this warp or
        // start before a row's window (warp-uniform).
        if (t0 + kN - 1 > wr0 || (p.window > 0 && t0 < first_key(wr1, p.window))) {
#pragma unroll
          for (int c = 0; c < kN; ++c) {
            const int kp = t0 + c;
            if (kp > pr || kp < lo) sv[c] = __float_as_uint(-INFINITY);
          }
        }
        // four independent running maxima of three inputs each (two keys a step),
        // then their maximum: 64 instructions for 128 keys, short chains
        auto sf = [&](int c) { return __uint_as_float(sv[c]); };
        float mxa = sf(0), mxb = sf(1), mxc = sf(2), mxd = sf(3);
#pragma unroll
        for (int c = 4; c + 8 <= kN - 4; c += 8) {
          mxa = fmax3f(mxa, sf(c), sf(c + 1));
          mxb = fmax3f(mxb, sf(c + 2), sf(c + 3));
          mxc = fmax3f(mxc, sf(c + 4), sf(c + 5));
          mxd = fmax3f(mxd, sf(c + 6), sf(c + 7));
        }
        mxa = fmax3f(mxa, sf(kN - 4), sf(kN - 3));
        mxb = fmax3f(mxb, sf(kN - 2), sf(kN - 1));
        const float mx = fmax3f(mxa, mxb, fmaxf(mxc, mxd)) * p.scale_log2;  // log2 domain
        // move the reference max when it grew past the lazy bound; O and l are
        // rescaled below, once this tile's scores are no longer held in registers
        const bool grow =
            mx > m_ref + t5::kLazyRescale || (m_ref == -INFINITY && mx > -INFINITY);
        const bool rescale = __any_sync(0xffffffffu, grow && m_ref > -INFINITY);
        const float alpha = grow && m_ref > -INFINITY ? exp2f(m_ref - mx) : 1.f;
        if (grow) m_ref = mx;
        const float nbase = m_ref == -INFINITY ? 0.f : -m_ref;
        // this tile's P row, weight = 2^(s * scale_log2 - m_ref) (one FMA per key, two
        // keys per instruction, and one exp2 per key), packed two per column over the
        // first half of its S row, in halves of 64 keys (each half's 32 columns stored
        // at once); l sums the same rounded weights the product uses, in four partial
        // sums, each 16-bit weight added as it is (mixed-precision add)
        const uint64_t scale2 = f32x2(p.scale_log2, p.scale_log2), base2 = f32x2(nbase, nbase);
        float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c4 = 0; c4 < kN / 64; ++c4) {
          uint32_t pw[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int kx = c4 * 64 + 2 * c;
            float xa, xb;
            f32x2_split(fma_f32x2(f32x2(sf(kx), sf(kx + 1)), scale2, base2), xa, xb);
            float ra, rb;
            pw[c] = Mma<T>::pack(ex2_approx(xa), ex2_approx(xb), ra, rb);
            Mma<T>::add_halves(ls4[c % 4], pw[c]);
          }
          tmem_st32(trow + c4 * 32, pw);
        }
        l = l * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));
        // O against the new reference max (warp-uniform TMEM traffic: lanes that keep
        // theirs scale by 1), before this tile's P V is issued. S was issued after
        // the group's previous P V and the tensor core runs in order, so O holds it.
        if (rescale) {
          wait_bounded(pv_done(grp), (t - 1) & 1, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32(trow + 128 + c4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(trow + 128 + c4 * 32, o);
          }
        }
        // rows of V outside every row's keys may hold anything: zero them (both
        // groups zero the same rows of a shared slot; the writes are identical)
        const int nvalid = min(kN, n - t0);
        const int nskip = max(0, lo_first - t0);
        if (nvalid < kN || nskip > 0) {
          const long long gv = vg + j;
          // (after the TMA copies into this V slot have landed)
          wait_bounded(&v_full[gv % NV], (gv / NV) & 1, abort_flag);
          unsigned char *vz = smem + L::kVRingOff + (gv % NV) * L::kSlotBytes;
          // rows [0, nskip) and [max(nvalid, nskip), kN): only those rows are visited
          const int hi0 = max(nvalid, nskip);
          const int nrows = nskip + (kN - hi0);
          for (int c = r; c < nrows * 8 * L::kPanels; c += 128) {
            const int i = c / (8 * L::kPanels), pn = (c / 8) % L::kPanels, ch = c % 8;
            const int vr = i < nskip ? i : hi0 + (i - nskip);
            *reinterpret_cast<uint4 *>(vz + pn * L::kKVPanel + vr * 128 + (ch << 4)) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(grp));
      }
      // ---- O / l -> global memory, then O goes back to the issuing thread
      if (my_tiles > 0) {
        wait_bounded(pv_done(grp), (tg + my_tiles - 1) & 1, abort_flag);
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        T *og = static_cast<T *>(p.out);
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t o[32];
          tmem_ld32(trow + 128 + c4 * 32, o);
          tmem_wait_ld();
          if (R < rows) {
            uint4 *dst = reinterpret_cast<uint4 *>(
                og + ((size_t)(I.qs0 + I.q0 + R) * p.num_q_heads + I.h + grp * g_head) * D +
                c4 * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t w[4];
              float a, c;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = Mma<T>::pack(__uint_as_float(o[q4 * 8 + 2 * e]) * inv,
                                    __uint_as_float(o[q4 * 8 + 2 * e + 1]) * inv, a, c);
              dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_free(grp));
      tg += my_tiles;
      vg += I.ntiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, t5::kTmemCols);
}

template <typename T, int D>
pa_status launch(const PrefillParams &prm, const void *k_cache, const void *v_cache,
                 pa_dtype dtype, cudaStream_t stream) {
  using L = Layout<D>;
  CUtensorMap tk, tv;
  constexpr int kKTile = 64;  // keys per stage
  const long long rows = (long long)prm.num_blocks * prm.num_kv_heads * prm.block_size;
  const int box_rows = prm.block_size < kKTile ? prm.block_size : kKTile;
  if (!pa_internal_pool_tensor_map(&tk, k_cache, rows, D, box_rows, dtype) ||
      !pa_internal_pool_tensor_map(&tv, v_cache, rows, D, box_rows, dtype))
    return PA_ERR_CUDA;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(pa_prefill_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kBytes) != cudaSuccess)
      return PA_ERR_CUDA;
    configured[dev] = true;
  }
  dim3 grid((unsigned)prm.num_q_heads, (unsigned)prm.q_tiles, (unsigned)prm.num_seqs);
  pa_prefill_kernel<T, D><<<grid, kThreads, L::kBytes, stream>>>(tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The persistent kernel's work counter and item order: one of each per device,
// written on the stream before every launch. Only a successful address lookup is
// kept.
__device__ unsigned g_prefill_work;

constexpr int kOrderThreads = 1024;
constexpr int kOrderBuckets = 1024;  // tile counts from the last bucket on share it
constexpr int kOrderCap = 16384;     // (sequence, query tile) pairs the order holds
__device__ int g_prefill_order[kOrderCap];

template <typename Sym>
void *symbol_address(const Sym &sym, void **cache) {
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void *a = nullptr;
    if (cudaGetSymbolAddress(&a, sym) != cudaSuccess || !a) {
      cudaGetLastError();
      return nullptr;
    }
    cache[dev] = a;
  }
  return cache[dev];
}

unsigned *prefill_work_counter() {
  static void *addr[64] = {};
  return static_cast<unsigned *>(symbol_address(g_prefill_work, addr));
}

int *prefill_order_buffer() {
  static void *addr[64] = {};
  return static_cast<int *>(symbol_address(g_prefill_order, addr));
}

// The order in which the persistent kernel's CTAs take the (sequence, query tile)
// pairs: by the number of key tiles the pair's items read, most first, so that the
// last items the CTAs take are short ones and the CTAs finish close together (the
// longest-processing-time-first rule of list scheduling). One CTA: a counting sort
// over the tile count (pairs with equal counts in any order; which CTA computes an
// item, and when, does not change its result). It also clears the work counter.
__global__ void __launch_bounds__(kOrderThreads) prefill_order_kernel(const PrefillParams p,
                                                                     int *order, unsigned *work) {
  __shared__ int hist[kOrderBuckets];
  __shared__ int warp_base[kOrderThreads / 32];
  // the persistent kernel behind this one may start its set-up now; it reads the
  // order and the counter only once this kernel has completed (griddepcontrol.wait)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) *work = 0u;
  for (int i = tid; i < kOrderBuckets; i += kOrderThreads) hist[i] = 0;
  __syncthreads();
  const int pairs = p.num_seqs * p.q_tiles;
  const int item_rows = p.pair_heads ? t5::kM : t5::kGroups * t5::kM;
  const int align = p.block_size < t5::kN ? p.block_size : t5::kN;
  const int cap = p.max_blocks_per_seq * p.block_size;
  // the item's tiles as the persistent kernel counts them (lengths clamped the same
  // way), as a bucket index that grows as the count falls
  auto bucket_of = [&](int u) {
    const int b = u / p.q_tiles;
    const int qt = p.q_tiles - 1 - u % p.q_tiles;
    const int n = max(0, min(min(__ldg(p.context_lens + b), cap), p.max_context_len));
    const int qs0 = __ldg(p.q_start + b), qs1 = __ldg(p.q_start + b + 1);
    int m = qs1 - qs0;
    if (m < 0 || m > n || qs0 < 0 || qs1 > p.num_tokens) m = 0;
    const int q0 = qt * item_rows;
    const int rows = m > q0 ? min(item_rows, m - q0) : 0;
    const int p_first = n - m + q0;
    const int k_base = first_key(p_first, p.window) & ~(align - 1);
    const int tiles = rows > 0 ? (p_first + rows - k_base + t5::kN - 1) / t5::kN : 0;
    return kOrderBuckets - 1 - min(tiles, kOrderBuckets - 1);
  };
  for (int u = tid; u < pairs; u += kOrderThreads) atomicAdd(&hist[bucket_of(u)], 1);
  __syncthreads();
  // bucket starts: an exclusive prefix sum over the buckets, kPer per thread
  constexpr int kPer = kOrderBuckets / kOrderThreads;
  int cnt[kPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    cnt[i] = hist[tid * kPer + i];
    sum += cnt[i];
  }
  int incl = sum;
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_base[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_base[lane];
    int wi = w;
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += v;
    }
    warp_base[lane] = wi - w;
  }
  __syncthreads();
  int start = warp_base[warp] + incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    hist[tid * kPer + i] = start;
    start += cnt[i];
  }
  __syncthreads();
  for (int u = tid; u < pairs; u += kOrderThreads) order[atomicAdd(&hist[bucket_of(u)], 1)] = u;
}

// TMA tensor map over q viewed as [num_tokens][num_q_heads][head_dim]: boxes of 64
// head_dim columns x 1 head x 128 tokens (the rows of one group),
// 128-byte swizzle; tokens past num_tokens read as zeros. Cached per (base, shape).
bool q_tensor_map(CUtensorMap *map, const void *q, int num_tokens, int num_q_heads, int head_dim,
                  pa_dtype dtype) {
  struct Key {
    const void *q;
    int t, h, d, dt;
  };
  constexpr int kSlots = 16;
  static std::mutex mu;
  static Key keys[kSlots];
  static CUtensorMap maps[kSlots];
  static int used = 0, next = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (keys[i].q == q && keys[i].t == num_tokens && keys[i].h == num_q_heads &&
        keys[i].d == head_dim && keys[i].dt == (int)dtype) {
      *map = maps[i];
      return true;
    }
  using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion,
                                     CUtensorMapFloatOOBfill);
  static EncodeTiledFn enc = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads,
                              (cuuint64_t)num_tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2,
                                 (cuuint64_t)num_q_heads * head_dim * 2};
  const cuuint32_t box[3] = {64u, 1u, (cuuint32_t)t5::kM};  // one group's rows
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUtensorMap m;
  if (enc(&m, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
          3, const_cast<void *>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = used < kSlots ? used++ : (next++ % kSlots);
  keys[slot] = Key{q, num_tokens, num_q_heads, head_dim, (int)dtype};
  maps[slot] = m;
  *map = m;
  return true;
}

template <typename T, int D>
pa_status launch_tc(const PrefillParams &prm_in, int max_q_len, const void *k_cache,
                    const void *v_cache, pa_dtype dtype, cudaStream_t stream) {
  using L = t5::Lay<D>;
  PrefillParams prm = prm_in;
  // two q heads of one kv head per item where the heads pair up, else 256 rows of one
  prm.pair_heads = (prm.num_q_heads / prm.num_kv_heads) % 2 == 0 ? 1 : 0;
  const int item_rows = prm.pair_heads ? t5::kM : t5::kGroups * t5::kM;
  prm.q_tiles = (max_q_len + item_rows - 1) / item_rows;
  CUtensorMap tk, tv, tq;
  const long long rows = (long long)prm.num_blocks * prm.num_kv_heads * prm.block_size;
  const int box_rows = prm.block_size < t5::kN ? prm.block_size : t5::kN;
  if (!pa_internal_pool_tensor_map(&tk, k_cache, rows, D, box_rows, dtype) ||
      !pa_internal_pool_tensor_map(&tv, v_cache, rows, D, box_rows, dtype) ||
      !q_tensor_map(&tq, prm.q, prm.num_tokens, prm.num_q_heads, D, dtype))
    return PA_ERR_CUDA;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(pa_prefill_tc_kernel<T, D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
      return PA_ERR_CUDA;
    configured[dev] = true;
  }
  unsigned *work = prefill_work_counter();
  if (!work) return PA_ERR_CUDA;
  // one CTA per SM (a CTA fills an SM's shared and tensor memory), never more than items
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return PA_ERR_CUDA;
  const long long n_items =
      (long long)(prm.pair_heads ? prm.num_q_heads / 2 : prm.num_q_heads) * prm.q_tiles *
      prm.num_seqs;
  const unsigned grid = (unsigned)std::min<long long>(n_items, sms);
  // the item order (which also clears the counter), or index order past its capacity
  prm.order = nullptr;
  if ((long long)prm.num_seqs * prm.q_tiles <= kOrderCap) {
    int *order = prefill_order_buffer();
    if (!order) return PA_ERR_CUDA;
    prefill_order_kernel<<<1, kOrderThreads, 0, stream>>>(prm, order, work);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    prm.order = order;
  } else if (cudaMemsetAsync(work, 0, sizeof(unsigned), stream) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  // behind the order kernel: a programmatic dependent (its set-up overlaps that kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(t5::kThreads);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = prm.order ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, pa_prefill_tc_kernel<T, D>, tk, tv, tq, prm, work) != cudaSuccess)
    return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

}  // namespace

extern "C" pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, const int32_t *q_start,
                                int num_seqs, int num_tokens, int max_q_len,
                                int max_context_len, int num_q_heads, int num_kv_heads,
                                int head_dim, int block_size, int num_blocks, float scale,
                                int window, pa_dtype dtype, void *stream) {
  if (num_seqs < 0 || num_tokens < 0 || max_q_len < 0 || max_context_len < 0 || window < 0 ||
      num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads || block_size <= 0 ||
      num_blocks <= 0 || max_blocks_per_seq <= 0 || (dtype != PA_F16 && dtype != PA_BF16))
    return PA_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  // TMA boxes are whole blocks or 64-key slices of one
  if (block_size < 8 || (block_size & (block_size - 1))) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_tokens == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !q_start)
    return PA_ERR_INVALID;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(q_start, 4))
    return PA_ERR_INVALID;
  const long long rows = (long long)num_blocks * num_kv_heads * block_size;
  if (rows > INT32_MAX || num_seqs > 65535 || num_q_heads > 65535) return PA_ERR_INVALID;
  const int q_tiles = (max_q_len + kQTile - 1) / kQTile;
  if (q_tiles > 65535) return PA_ERR_INVALID;
  PrefillParams prm;
  prm.out = out;
  prm.q = q;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.q_start = q_start;
  prm.max_blocks_per_seq = max_blocks_per_seq;
  prm.max_context_len = max_context_len;
  prm.num_tokens = num_tokens;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.window = window;
  prm.q_tiles = q_tiles;
  prm.pair_heads = 0;
  prm.order = nullptr;
  prm.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#if PA_PREFILL_TCGEN05
  if (dtype == PA_BF16)
    return head_dim == 128 ? launch_tc<__nv_bfloat16, 128>(prm, max_q_len, k_cache, v_cache, dtype, st)
                           : launch_tc<__nv_bfloat16, 64>(prm, max_q_len, k_cache, v_cache, dtype, st);
  return head_dim == 128 ? launch_tc<__half, 128>(prm, max_q_len, k_cache, v_cache, dtype, st)
                         : launch_tc<__half, 64>(prm, max_q_len, k_cache, v_cache, dtype, st);
#else
  if (dtype == PA_BF16)
    return head_dim == 128 ? launch<__nv_bfloat16, 128>(prm, k_cache, v_cache, dtype, st)
                           : launch<__nv_bfloat16, 64>(prm, k_cache, v_cache, dtype, st);
  return head_dim == 128 ? launch<__half, 128>(prm, k_cache, v_cache, dtype, st)
                         : launch<__half, 64>(prm, k_cache, v_cache, dtype, st);
#endif
}

// Read and clear this file's error word (stream-ordered; synchronises the stream).
pa_status pa_internal_prefill_status(cudaStream_t stream, int32_t *code) {
  int value = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&value, g_prefill_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_prefill_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                              stream) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
  *code = value;
  return PA_OK;
}
