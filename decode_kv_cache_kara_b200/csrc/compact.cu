// Paged compaction: Kara's compressed windows and LaCache's ladder, through one gather.
//
// "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression", English
// abstract: Kara is adapted to PagedAttention; the kept KV pairs move into fresh blocks, the
// block table is rewritten and the old blocks are freed. "LaCache: Ladder-Shaped KV Caching
// ...": states outside the ladder are dropped and the rest packed into a smaller cache
// (method details), re-applied when the cache is full (iterative compaction).
//
// Stream-ordered kernels per call:
//   check    (kara_compact only, a few CTAs) checks the caller's keep sets: every entry a
//                        window position, every row strictly ascending; the plan reads the
//                        verdicts and refuses the whole call on a bad entry.
//   plan     (one CTA)   validates every due sequence, computes its page geometry and pops its
//                        fresh blocks from the free list (sequence order, stack top first); on
//                        any error it records the status and marks the plan invalid.
//   gather   (wide grid, launched as a programmatic dependent of the plan) copies rows with
//                        16-byte loads/stores, all of a thread's rows in flight at once:
//                        sources through the old block table, destinations into the fresh
//                        blocks. Kara copies one KV head's row per kept position; LaCache copies
//                        whole [Hkv, d] rows of the ladder's kept slots (computed analytically
//                        per layer). Per sequence, the CTA that finishes last (a counter in
//                        the sequence's plan row, zeroed by the plan) rewrites the sequence's
//                        block table entries, pushes its old blocks and sets its ctx_len;
//                        every CTA that reads that sequence's old table entries is done by
//                        then. The plan sets free_top (nothing later in the call reads it).
// The gather reads only blocks that belong to the sequences and writes only fresh blocks, so
// sources never alias destinations; nothing is modified unless the plan is valid.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "select_row.cuh"

namespace kara {

namespace {

constexpr int kPlanThreads = 1024;
// Header: [0..4) valid, total_new, total_old, top; [16, 16 + kCheckCtas) the verdicts of the
// keep check's CTAs (nonzero = a bad entry in that CTA's rows)
constexpr int kCheckCtas = 128;
constexpr int kCheckThreads = 512;
constexpr int kHdrCheck = 16;
constexpr int kPlanHeader = kHdrCheck + kCheckCtas;
constexpr int kPlanStride = 12;   // b, n, start, off, p0, n_old, n_new, base_new, base_old, done
enum { P_B = 0, P_N, P_START, P_OFF, P_P0, P_NOLD, P_NNEW, P_BNEW, P_BOLD, P_DONE };


struct PlanParams {
  const int32_t* block_table;
  const int32_t* ctx_len;
  const int32_t* free_list;
  int32_t* free_top;
  const int32_t* seq_ids;
  int32_t* plan;
  int32_t* status;
  int R, batch, max_blocks, num_blocks;
  // Kara: window W and budget k. LaCache: W = 0, k = budget, min_len = sink+recent+R_max.
  int W, k, lacache, min_len;
  int check_ctas;   // CTAs of the keep check that ran before the plan (0: no check)
};

// The caller's keep sets, before anything is planned: every entry of every (layer, sequence,
// KV head) row must be a window position (0 <= pos < W) and each row strictly ascending.
// Each CTA writes its verdict to its own header slot (so nothing has to be cleared first);
// the plan refuses the call, moving and freeing nothing, when any verdict is nonzero.
struct KeepCheck {
  const int32_t* keep;
  int32_t* plan;
  long long rows;
  int k, W;
};

__global__ void __launch_bounds__(kCheckThreads) keep_check_kernel(const KeepCheck c) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // keep is complete (PDL launch)
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  constexpr int kWarps = kCheckThreads / 32;
  int bad = 0;
  for (long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
       row < c.rows; row += static_cast<long long>(gridDim.x) * kWarps) {
    const int32_t* kr = c.keep + row * c.k;
    for (int t = lane; t < c.k; t += 32) {
      const int pos = kr[t];
      if (pos < 0 || pos >= c.W || (t > 0 && kr[t - 1] >= pos)) bad = 1;
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (threadIdx.x == 0) c.plan[kHdrCheck + blockIdx.x] = s_bad;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  __shared__ int buf[33];
  __shared__ int err;
  __shared__ int carry_new, carry_old;
  int32_t* hdr = p.plan;
  int32_t* rows = p.plan + kPlanHeader;
  int32_t* fresh = rows + static_cast<size_t>(p.R) * kPlanStride;
  __shared__ int s_top;
  if (threadIdx.x == 0) {
    err = 0;
    carry_new = 0;
    carry_old = 0;
    s_top = *p.free_top;     // read once, early: thread 0 also writes the new top below
  }
  __syncthreads();
  // the gather may be scheduled now; it waits for this grid's results itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // 1. geometry of every due sequence, exclusive scans of its fresh / old page counts
  for (int base = 0; base < p.R; base += kPlanThreads) {
    const int r = base + threadIdx.x;
    int n_new = 0, n_old = 0;
    if (r < p.R) {
      int code = 0;
      const int b = p.seq_ids ? p.seq_ids[r] : r;
      if (b < 0 || b >= p.batch) code = KARA_ERR_INVALID_ARG;
      if (!code && p.seq_ids && r > 0 && p.seq_ids[r - 1] >= b) code = KARA_ERR_INVALID_ARG;
      const int n = code ? 0 : p.ctx_len[b];
      int start = 0, off = 0, p0 = 0;
      if (!code) {
        if (p.lacache) {
          if (n < p.min_len || n > p.max_blocks * 16) code = KARA_ERR_INVALID_ARG;
          n_old = (n + 15) / 16;
          n_new = (p.k + 15) / 16;
        } else {
          if (n < p.W || n > p.max_blocks * 16) code = KARA_ERR_INVALID_ARG;
          start = n - p.W;
          off = start % 16;
          p0 = start / 16;
          n_old = (off + p.W + 15) / 16;
          n_new = (off + p.k + 15) / 16;
        }
      }
      if (code) {
        atomicCAS(&err, 0, code);
        n_new = n_old = 0;
      }
      int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
      row[P_B] = b;
      row[P_N] = n;
      row[P_START] = start;
      row[P_OFF] = off;
      row[P_P0] = p0;
      row[P_NOLD] = n_old;
      row[P_NNEW] = n_new;
      row[P_DONE] = 0;     // gather CTAs of this sequence done
    }
    int tot_new, tot_old;
    const int ex_new = block_scan_add(n_new, buf, &tot_new);
    const int ex_old = block_scan_add(n_old, buf, &tot_old);
    if (r < p.R) {
      int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
      row[P_BNEW] = carry_new + ex_new;
      row[P_BOLD] = carry_old + ex_old;
    }
    __syncthreads();
    if (threadIdx.x == 0) { carry_new += tot_new; carry_old += tot_old; }
    __syncthreads();
  }
  // 2. every old page id of every due sequence must be a valid block (a warp per sequence);
  // the fresh blocks are popped at the same time (sequence order, stack top first; they are
  // used only if the plan turns out valid)
  {
    const int top = s_top;
    if (top >= 0 && top <= p.num_blocks && carry_new <= top)
      for (int i = threadIdx.x; i < carry_new; i += kPlanThreads) fresh[i] = p.free_list[top - 1 - i];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < p.check_ctas && hdr[kHdrCheck + threadIdx.x] != 0)
      atomicCAS(&err, 0, KARA_ERR_INVALID_ARG);     // a keep entry outside the window
    for (int r = warp; r < p.R; r += kPlanThreads / 32) {
      const int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
      const int n_old = row[P_NOLD];
      const int32_t* tab = p.block_table + static_cast<size_t>(row[P_B]) * p.max_blocks + row[P_P0];
      for (int pg = lane; pg < n_old; pg += 32) {
        const int blk = tab[pg];
        if (blk < 0 || blk >= p.num_blocks) atomicCAS(&err, 0, KARA_ERR_BAD_BLOCK);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int top = s_top;
    int code = err;
    if (!code && (top < 0 || top > p.num_blocks)) code = KARA_ERR_INVALID_ARG;
    if (!code && carry_new > top) code = KARA_ERR_OUT_OF_BLOCKS;
    // the pushes must fit: an inconsistent free list (ids still in use) is refused
    if (!code && top - carry_new + carry_old > p.num_blocks) code = KARA_ERR_INVALID_ARG;
    if (code) report(p.status, code);
    hdr[0] = code ? 0 : 1;
    hdr[1] = carry_new;
    hdr[2] = carry_old;
    hdr[3] = top;
    // pops [top - new, top), pushes [top - new, top - new + old): the final top
    if (!code) *p.free_top = top - carry_new + carry_old;
    err = code;
  }
}

struct FinalizeParams {
  int32_t* block_table;
  int32_t* ctx_len;
  int32_t* free_list;
  int32_t* plan;
  int R, max_blocks, k;   // k: kept slots (Kara) or budget (LaCache)
};

// Called by every thread of each gather CTA when its copies are done; `per_seq` CTAs work on
// sequence row r. The last of them rewrites the sequence's table entries of its old pages
// (fresh id or -1), pushes the old ids onto the free list and sets the sequence's ctx_len.
// `s_old` / `s_fresh`: the sequence's old and fresh ids staged in shared memory (or null).
__device__ void finalize_if_last(const FinalizeParams& p, int r, int per_seq,
                                 const int* s_old = nullptr, const int* s_fresh = nullptr) {
  __shared__ int s_last;
  int32_t* row = p.plan + kPlanHeader + static_cast<size_t>(r) * kPlanStride;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&row[P_DONE], 1) == per_seq - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int32_t* hdr = p.plan;
  const int32_t* fresh = p.plan + kPlanHeader + static_cast<size_t>(p.R) * kPlanStride;
  const int push_base = hdr[3] - hdr[1];
  const int n_old = row[P_NOLD], n_new = row[P_NNEW], bnew = row[P_BNEW], bold = row[P_BOLD];
  int32_t* tab = p.block_table + static_cast<size_t>(row[P_B]) * p.max_blocks + row[P_P0];
  for (int pg = threadIdx.x; pg < n_old; pg += blockDim.x) {
    const int old = s_old ? s_old[pg] : tab[pg];
    tab[pg] = pg < n_new ? (s_fresh ? s_fresh[pg] : fresh[bnew + pg]) : -1;
    p.free_list[push_base + bold + pg] = old;
  }
  if (threadIdx.x == 0 && n_old > 0) p.ctx_len[row[P_B]] = row[P_START] + p.k;
}

// ------------------------------------------------------------------------------------------
// Kara gather: CTA = (layer, sequence, KV head, chunk of kept rows). Chunk 0 also copies the
// prefix rows of the first window page for its head.
// ------------------------------------------------------------------------------------------
constexpr int kGatherThreads = 128;
constexpr int kChunkRows = 256;

struct KaraGather {
  LayerPtrs layers;
  const int32_t* block_table;
  const int32_t* keep;
  const int32_t* plan;
  int32_t* status;
  int R, Hkv, k, W, max_blocks;
  FinalizeParams fin;
};

// Pages a window can span (KARA_MAX_WINDOW slots at any slot offset), plus one.
constexpr int kMaxWindowPages = (KARA_MAX_WINDOW + 15 + 15) / 16 + 1;

template <int D>
__global__ void __launch_bounds__(kGatherThreads) kara_gather_kernel(const KaraGather g) {
  __shared__ int s_old[kMaxWindowPages];     // old block ids of the window's pages
  __shared__ int s_fresh[kMaxWindowPages];   // the sequence's fresh block ids
  __shared__ int s_keep[kChunkRows];         // this chunk's kept positions
  // the CTA's rows (prefix rows, then kept rows): source and destination row starts in
  // 16-byte units, once per row rather than per piece; ~0 marks a row that is not copied
  __shared__ size_t s_src[kChunkRows + 16], s_dst[kChunkRows + 16];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int32_t* hdr = g.plan;
  if (hdr[0] != 1) return;
  constexpr int kVecPerRow = D * 2 / 16;                  // 16-byte pieces per head row
  constexpr int kRowsPerPass = kGatherThreads / kVecPerRow;
  const int chunk = blockIdx.x;
  const int head = blockIdx.y % g.Hkv;
  const int r = blockIdx.y / g.Hkv;
  const int layer = blockIdx.z;
  const int32_t* rows = g.plan + kPlanHeader;
  const int32_t* fresh = rows + static_cast<size_t>(g.R) * kPlanStride;
  const int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
  const int b = row[P_B], start = row[P_START], off = row[P_OFF], p0 = row[P_P0];
  const int n_old = row[P_NOLD], n_new = row[P_NNEW];
  const int t0 = chunk * kChunkRows;
  const int t1 = min(g.k, t0 + kChunkRows);
  // one round trip for every index this CTA needs
  const int32_t* tab = g.block_table + static_cast<size_t>(b) * g.max_blocks + p0;
  const int32_t* fr = fresh + row[P_BNEW];
  const int32_t* kp = g.keep + ((static_cast<size_t>(layer) * g.R + r) * g.Hkv + head) * g.k;
  for (int i = threadIdx.x; i < n_old; i += kGatherThreads) s_old[i] = tab[i];
  for (int i = threadIdx.x; i < n_new; i += kGatherThreads) s_fresh[i] = fr[i];
  for (int i = threadIdx.x; i < t1 - t0; i += kGatherThreads) s_keep[i] = kp[t0 + i];
  __syncthreads();
  // rows handled by this CTA: prefix rows (chunk 0 only), then kept rows of the chunk
  const int npre = (chunk == 0) ? off : 0;
  const int total = npre + max(0, t1 - t0);
  for (int i = threadIdx.x; i < total; i += kGatherThreads) {
    int src_slot, dst_slot;
    bool ok = true;
    if (i < npre) {
      src_slot = dst_slot = p0 * 16 + i;
    } else {
      const int pos = s_keep[i - npre];
      ok = pos >= 0 && pos < g.W;          // refused by the plan already; never read outside
      src_slot = start + (ok ? pos : 0);
      dst_slot = start + t0 + (i - npre);
    }
    const int sblk = s_old[(src_slot >> 4) - p0];
    const int dblk = s_fresh[(dst_slot >> 4) - p0];
    s_src[i] = ok ? ((static_cast<size_t>(sblk) * 16 + (src_slot & 15)) * g.Hkv + head) * kVecPerRow
                  : ~size_t(0);
    s_dst[i] = ((static_cast<size_t>(dblk) * 16 + (dst_slot & 15)) * g.Hkv + head) * kVecPerRow;
  }
  __syncthreads();
  const uint4* ksrc = reinterpret_cast<const uint4*>(g.layers.k[layer]);
  const uint4* vsrc = reinterpret_cast<const uint4*>(g.layers.v[layer]);
  uint4* kdst = reinterpret_cast<uint4*>(g.layers.k[layer]);
  uint4* vdst = reinterpret_cast<uint4*>(g.layers.v[layer]);
  const int vec = threadIdx.x % kVecPerRow;
  const int sub = threadIdx.x / kVecPerRow;
  constexpr int kUnroll = 8;
  for (int base = sub; base < total; base += kRowsPerPass * kUnroll) {
    uint4 kv[kUnroll], vv[kUnroll];
    size_t dsti[kUnroll];
    bool act[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + u * kRowsPerPass;
      act[u] = i < total && s_src[i] != ~size_t(0);
      if (!act[u]) continue;
      const size_t si = s_src[i] + vec;
      dsti[u] = s_dst[i] + vec;
      kv[u] = ksrc[si];
      vv[u] = vsrc[si];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!act[u]) continue;
      kdst[dsti[u]] = kv[u];
      vdst[dsti[u]] = vv[u];
    }
  }
  finalize_if_last(g.fin, r, gridDim.x * g.Hkv * gridDim.z, s_old, s_fresh);
}

// ------------------------------------------------------------------------------------------
// Fused compression: CTA = (layer, sequence, KV head) of kSelThreads threads. The compaction
// plan depends only on (n, W, k) of each sequence, not on which positions are kept, so it
// runs first; each CTA then selects and expands its row in shared memory (select_row.cuh),
// copies the head's prefix rows of the first window page and its k kept rows into the fresh
// blocks, and the sequence's last CTA finalizes it. keep_out (optional) gets the keep sets.
// ------------------------------------------------------------------------------------------
struct CompressArgs {
  KaraGather g;                  // g.keep unused
  const float* scores;           // [L, R, Hkv, W]
  int32_t* keep_out;             // [L, R, Hkv, k] or null
  int num_anchors, gap_limit, widen;
};

__host__ __device__ constexpr size_t compress_keep_off(int W) {
  return (t2c_smem(W) + 15) / 16 * 16;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) compress_kernel(const CompressArgs c) {
  __shared__ int s_old[kMaxWindowPages];
  __shared__ int s_fresh[kMaxWindowPages];
  extern __shared__ __align__(16) uint8_t dsm[];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const KaraGather& g = c.g;
  const int head = blockIdx.y % g.Hkv;
  const int r = blockIdx.y / g.Hkv;
  const int layer = blockIdx.z;
  const size_t rowi = (static_cast<size_t>(layer) * g.R + r) * g.Hkv + head;
  int32_t* s_keep = reinterpret_cast<int32_t*>(dsm + compress_keep_off(g.W));
  // 1. selection and Token2Chunk of the row, the keep set into shared memory
  token2chunk_row(c.scores + rowi * g.W, nullptr, nullptr, g.W, g.k, c.num_anchors,
                  c.gap_limit, c.widen, s_keep, dsm);
  __syncthreads();
  if (c.keep_out != nullptr)
    for (int i = threadIdx.x; i < g.k; i += kSelThreads) c.keep_out[rowi * g.k + i] = s_keep[i];
  const int32_t* hdr = g.plan;
  if (hdr[0] != 1) return;        // the plan refused (and reported): nothing moves
  // 2. the gather of the row's prefix rows and kept rows
  constexpr int kVecPerRow = D * 2 / 16;
  constexpr int kRowsPerPass = kSelThreads / kVecPerRow;
  const int32_t* rows = g.plan + kPlanHeader;
  const int32_t* fresh = rows + static_cast<size_t>(g.R) * kPlanStride;
  const int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
  const int b = row[P_B], start = row[P_START], off = row[P_OFF], p0 = row[P_P0];
  const int n_old = row[P_NOLD], n_new = row[P_NNEW];
  const int32_t* tab = g.block_table + static_cast<size_t>(b) * g.max_blocks + p0;
  const int32_t* fr = fresh + row[P_BNEW];
  for (int i = threadIdx.x; i < n_old; i += kSelThreads) s_old[i] = tab[i];
  for (int i = threadIdx.x; i < n_new; i += kSelThreads) s_fresh[i] = fr[i];
  __syncthreads();
  const uint4* ksrc = reinterpret_cast<const uint4*>(g.layers.k[layer]);
  const uint4* vsrc = reinterpret_cast<const uint4*>(g.layers.v[layer]);
  uint4* kdst = reinterpret_cast<uint4*>(g.layers.k[layer]);
  uint4* vdst = reinterpret_cast<uint4*>(g.layers.v[layer]);
  const int vec = threadIdx.x % kVecPerRow;
  const int sub = threadIdx.x / kVecPerRow;
  const int total = off + g.k;
  constexpr int kUnroll = 8;
  for (int base = sub; base < total; base += kRowsPerPass * kUnroll) {
    uint4 kv[kUnroll], vv[kUnroll];
    size_t dsti[kUnroll];
    bool act[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + u * kRowsPerPass;
      act[u] = i < total;
      if (!act[u]) continue;
      int src_slot, dst_slot;
      if (i < off) {
        src_slot = dst_slot = p0 * 16 + i;
      } else {
        src_slot = start + s_keep[i - off];
        dst_slot = start + (i - off);
      }
      const int sblk = s_old[(src_slot >> 4) - p0];
      const int dblk = s_fresh[(dst_slot >> 4) - p0];
      const size_t si = ((static_cast<size_t>(sblk) * 16 + (src_slot & 15)) * g.Hkv + head) *
                            kVecPerRow + vec;
      dsti[u] = ((static_cast<size_t>(dblk) * 16 + (dst_slot & 15)) * g.Hkv + head) *
                    kVecPerRow + vec;
      kv[u] = ksrc[si];
      vv[u] = vsrc[si];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!act[u]) continue;
      kdst[dsti[u]] = kv[u];
      vdst[dsti[u]] = vv[u];
    }
  }
  // 3. the sequence's last CTA (of L x Hkv) rewrites its table, frees its old blocks and
  // sets its length
  finalize_if_last(g.fin, r, g.Hkv * gridDim.z, s_old, s_fresh);
}

// ------------------------------------------------------------------------------------------
// LaCache gather: CTA = (layer, sequence, chunk of compacted slots); whole [Hkv, d] rows.
// ------------------------------------------------------------------------------------------
struct LadderGather {
  LayerPtrs layers;
  const int32_t* block_table;
  const int32_t* plan;
  int R, L, max_blocks;
  int row_vecs;          // 16-byte pieces per slot row (Hkv * D * 2 / 16)
  int span, overlap, rung, budget, sink, recent, r_max;
  FinalizeParams fin;
};

constexpr int kLadderSlots = 32;

// Source slot of compacted slot t in `layer`, for a sequence of n slots.
__device__ __forceinline__ int ladder_source(const LadderGather& g, int layer, int t, int n) {
  if (t < g.sink) return t;
  if (t >= g.budget - g.recent) return n - (g.budget - t);
  const int stride = g.span - g.overlap;
  const int q = g.span / stride;          // rungs one layer keeps per period
  const int period = g.L / stride;        // rungs per period
  const int tr = t - g.sink;
  const int per = tr / (q * g.rung);
  const int rem = tr % (q * g.rung);
  const int m = rem / g.rung;             // m-th kept rung of this layer within the period
  const int o = rem % g.rung;
  const int a = layer / stride;
  // kept rungs of the layer within a period: (a - u) mod period, u = 0..q-1, ascending
  int j;
  if (a >= q - 1) j = a - q + 1 + m;
  else j = (m <= a) ? m : period - q + m;
  const int region_start = n - g.recent - g.r_max;
  return region_start + (per * period + j) * g.rung + o;
}

__global__ void __launch_bounds__(kGatherThreads) ladder_gather_kernel(const LadderGather g) {
  __shared__ size_t s_src[kLadderSlots], s_dst[kLadderSlots];   // row starts, in 16-byte units
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int32_t* hdr = g.plan;
  if (hdr[0] != 1) return;
  const int chunk = blockIdx.x;
  const int r = blockIdx.y;
  const int layer = blockIdx.z;
  const int32_t* rows = g.plan + kPlanHeader;
  const int32_t* fresh = rows + static_cast<size_t>(g.R) * kPlanStride;
  const int32_t* row = rows + static_cast<size_t>(r) * kPlanStride;
  const int b = row[P_B], n = row[P_N];
  const int32_t* fr = fresh + row[P_BNEW];
  const int32_t* tab = g.block_table + static_cast<size_t>(b) * g.max_blocks;
  const uint4* ksrc = reinterpret_cast<const uint4*>(g.layers.k[layer]);
  const uint4* vsrc = reinterpret_cast<const uint4*>(g.layers.v[layer]);
  uint4* kdst = reinterpret_cast<uint4*>(g.layers.k[layer]);
  uint4* vdst = reinterpret_cast<uint4*>(g.layers.v[layer]);
  const int t0 = chunk * kLadderSlots;
  const int t1 = min(g.budget, t0 + kLadderSlots);
  // the chunk's source and destination rows, once per slot (not per 16-byte piece)
  if (threadIdx.x < t1 - t0) {
    const int t = t0 + threadIdx.x;
    const int src = ladder_source(g, layer, t, n);
    s_src[threadIdx.x] = (static_cast<size_t>(tab[src >> 4]) * 16 + (src & 15)) * g.row_vecs;
    s_dst[threadIdx.x] = (static_cast<size_t>(fr[t >> 4]) * 16 + (t & 15)) * g.row_vecs;
  }
  __syncthreads();
  const int pieces = (t1 - t0) * g.row_vecs;
  // row_vecs (Hkv * d * 2 / 16) is a power of two for power-of-two head counts: shifts then
  const bool pow2 = (g.row_vecs & (g.row_vecs - 1)) == 0;
  const int shift = __ffs(g.row_vecs) - 1;
  constexpr int kUnroll = 8;
  for (int base = threadIdx.x; base < pieces; base += kGatherThreads * kUnroll) {
    uint4 kv[kUnroll], vv[kUnroll];
    size_t dsti[kUnroll];
    bool act[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + u * kGatherThreads;
      act[u] = i < pieces;
      if (!act[u]) continue;
      const int tl = pow2 ? i >> shift : i / g.row_vecs;
      const int v = i - tl * g.row_vecs;
      const size_t si = s_src[tl] + v;
      dsti[u] = s_dst[tl] + v;
      kv[u] = ksrc[si];
      vv[u] = vsrc[si];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!act[u]) continue;
      kdst[dsti[u]] = kv[u];
      vdst[dsti[u]] = vv[u];
    }
  }
  finalize_if_last(g.fin, r, gridDim.x * gridDim.z);
}

// Launches `kernel` on `grid` x kGatherThreads as a programmatic dependent of the previous
// kernel in the stream (the plan).
template <typename Arg>
void launch_dependent(void (*kernel)(Arg), dim3 grid, const Arg& arg, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kGatherThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch(cudaLaunchKernelEx(&cfg, kernel, arg));
}

}  // namespace

size_t compact_workspace_bytes(int R, int W, int k) {
  (void)W;
  const size_t fresh = static_cast<size_t>(R) * ((15 + k + 15) / 16);
  return (kPlanHeader + static_cast<size_t>(R) * kPlanStride + fresh) * sizeof(int32_t);
}

size_t lacache_workspace_bytes(int R, int budget) {
  const size_t fresh = static_cast<size_t>(R) * ((budget + 15) / 16);
  return (kPlanHeader + static_cast<size_t>(R) * kPlanStride + fresh) * sizeof(int32_t);
}

kara_status launch_compact(const CompactLaunch& L, cudaStream_t stream) {
  if (L.R == 0) return KARA_OK;
  PlanParams pp;
  pp.block_table = L.block_table;
  pp.ctx_len = L.ctx_len;
  pp.free_list = L.free_list;
  pp.free_top = L.free_top;
  pp.seq_ids = L.seq_ids;
  pp.plan = L.plan;
  pp.status = L.status;
  pp.R = L.R;
  pp.batch = L.batch;
  pp.max_blocks = L.max_blocks;
  pp.num_blocks = L.num_blocks;
  pp.W = L.W;
  pp.k = L.k;
  pp.lacache = 0;
  pp.min_len = 0;
  pp.check_ctas = 0;
  if (L.scores == nullptr) {   // the caller's keep sets: checked before the plan
    KeepCheck kc;
    kc.keep = L.keep;
    kc.plan = L.plan;
    kc.rows = static_cast<long long>(L.L) * L.R * L.Hkv;
    kc.k = L.k;
    kc.W = L.W;
    const long long per_cta = kCheckThreads / 32;
    const int ctas = static_cast<int>(std::min<long long>(kCheckCtas, (kc.rows + per_cta - 1) / per_cta));
    launch_pdl(keep_check_kernel, dim3(ctas), dim3(kCheckThreads), 0, stream, kc);
    pp.check_ctas = ctas;
  }
  launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, pp);
  KaraGather g;
  g.layers = L.layers;
  g.block_table = L.block_table;
  g.keep = L.keep;
  g.plan = L.plan;
  g.status = L.status;
  g.R = L.R;
  g.Hkv = L.Hkv;
  g.k = L.k;
  g.W = L.W;
  g.max_blocks = L.max_blocks;
  g.fin.block_table = L.block_table;
  g.fin.ctx_len = L.ctx_len;
  g.fin.free_list = L.free_list;
  g.fin.plan = L.plan;
  g.fin.R = L.R;
  g.fin.max_blocks = L.max_blocks;
  g.fin.k = L.k;
  if (L.scores != nullptr) {
    CompressArgs c;
    c.g = g;
    c.scores = L.scores;
    c.keep_out = L.keep_out;
    c.num_anchors = L.num_anchors;
    c.gap_limit = L.gap_limit;
    c.widen = L.widen;
    const size_t smem = compress_keep_off(L.W) + static_cast<size_t>(L.k) * sizeof(int32_t);
    static std::atomic<int> attr_done[kMaxDevices];   // per device: the limit is set
    const int dev = device_slot();
    if (dev < 0) {
      set_last_error("kara_compress", "no usable current CUDA device");
      return KARA_ERR_CUDA;
    }
    if (!attr_done[dev].load()) {
      const int most = static_cast<int>(compress_keep_off(KARA_MAX_WINDOW) +
                                        KARA_MAX_WINDOW * sizeof(int32_t));
      cudaFuncSetAttribute(compress_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      cudaFuncSetAttribute(compress_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      attr_done[dev].store(1);
    }
    const dim3 grid(1, L.R * L.Hkv, L.L);
    if (L.D == 128) launch_pdl(compress_kernel<128>, grid, dim3(kSelThreads), smem, stream, c);
    else launch_pdl(compress_kernel<64>, grid, dim3(kSelThreads), smem, stream, c);
    return check_launch("kara_compress");
  }
  dim3 grid((L.k + kChunkRows - 1) / kChunkRows, L.R * L.Hkv, L.L);
  if (L.D == 128) launch_dependent(kara_gather_kernel<128>, grid, g, stream);
  else launch_dependent(kara_gather_kernel<64>, grid, g, stream);
  return check_launch(__func__);
}

kara_status launch_lacache(const LacacheLaunch& L, cudaStream_t stream) {
  if (L.R == 0) return KARA_OK;
  const int r_max = (L.budget - L.sink - L.recent) * L.L / L.span;
  PlanParams pp;
  pp.block_table = L.block_table;
  pp.ctx_len = L.ctx_len;
  pp.free_list = L.free_list;
  pp.free_top = L.free_top;
  pp.seq_ids = L.seq_ids;
  pp.plan = L.plan;
  pp.status = L.status;
  pp.R = L.R;
  pp.batch = L.batch;
  pp.max_blocks = L.max_blocks;
  pp.num_blocks = L.num_blocks;
  pp.W = 0;
  pp.k = L.budget;
  pp.lacache = 1;
  pp.min_len = L.sink + L.recent + r_max;
  pp.check_ctas = 0;
  launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, pp);
  LadderGather g;
  g.layers = L.layers;
  g.block_table = L.block_table;
  g.plan = L.plan;
  g.R = L.R;
  g.L = L.L;
  g.max_blocks = L.max_blocks;
  g.row_vecs = L.Hkv * L.D * 2 / 16;
  g.span = L.span;
  g.overlap = L.overlap;
  g.rung = L.rung;
  g.budget = L.budget;
  g.sink = L.sink;
  g.recent = L.recent;
  g.r_max = r_max;
  g.fin.block_table = L.block_table;
  g.fin.ctx_len = L.ctx_len;
  g.fin.free_list = L.free_list;
  g.fin.plan = L.plan;
  g.fin.R = L.R;
  g.fin.max_blocks = L.max_blocks;
  g.fin.k = L.budget;
  dim3 grid((L.budget + kLadderSlots - 1) / kLadderSlots, L.R, L.L);
  launch_dependent(ladder_gather_kernel, grid, g, stream);
  return check_launch(__func__);
}

}  // namespace kara

// ------------------------------------------------------------------------------------------
// kara_compact_noalloc: kara_compact with its plan scratch in a fixed device array.
//
// For callers that cannot allocate device memory when they compress: a serving engine that
// hands all free device memory to its KV block pool at start-up (a later cudaMalloc would
// fail, or would have to shrink the pool), and plain C callers that hold no device
// allocator. The caller still passes the pools, the bookkeeping and `keep`; only the plan
// (per-sequence geometry and the popped block ids) lives here.
// ------------------------------------------------------------------------------------------
namespace kara {
namespace {

constexpr size_t kNoAllocScratchBytes = KARA_COMPACT_NOALLOC_SCRATCH_BYTES;
// Every GPU that loads this library holds one copy of this array until the process exits.
static __device__ __align__(256) int32_t g_compact_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

std::mutex g_scratch_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device
// (in host code the array's name is only a host-side handle, not a device address).
kara_status scratch_for_current_device(int32_t** out) {
  const int dev = device_slot();
  if (dev < 0) return KARA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_compact_scratch) != cudaSuccess || p == nullptr)
      return KARA_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return KARA_OK;
}

}  // namespace
}  // namespace kara

extern "C" kara_status kara_compact_noalloc(const kara_layer_kv* layers, int32_t num_layers,
                                            const kara_pool* pool, const int32_t* seq_ids,
                                            int32_t num_seqs, int32_t window, int32_t k,
                                            const int32_t* keep, int32_t* dev_status,
                                            cudaStream_t stream) {
  using namespace kara;
  if (num_seqs < 0 || window < 1 || k < 1 || k > window) return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (compact_workspace_bytes(num_seqs, window, k) > kNoAllocScratchBytes)
    return KARA_ERR_WORKSPACE;   // the plan would not fit the fixed scratch array
  int32_t* scratch = nullptr;
  const kara_status st = scratch_for_current_device(&scratch);
  if (st != KARA_OK) return st;
  // The plan kernel writes every scratch entry it later reads, so nothing needs clearing.
  return kara_compact(layers, num_layers, pool, seq_ids, num_seqs, window, k, keep, scratch,
                      kNoAllocScratchBytes, dev_status, stream);
}
