// Block-level top-k selection and Token2Chunk of one window row, in shared memory: the device
// code of select.cu's kernels and of the fused compression kernel in compact.cu.
//
// Selection ("Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression",
// English abstract: select the informative KV pairs of the window): a most-significant-digit
// radix select over order-preserving 32-bit keys of the fp32 scores (4 passes of 8 bits,
// 256-bin shared-memory histograms), which finds the k-th largest key T exactly; positions
// above T are kept, and among positions equal to T the lowest ones, by a block-wide scan.
//
// Token2Chunk (same abstract: expand a subset of the selected KV pairs into chunks;
// gist.science explainer, section 2: the span between two important points is kept): anchors
// by the same radix select restricted to the selection; previous/next anchor and
// previous/next non-member positions by block-wide max/min scans over the window; gap fill,
// widening, run priorities and the trim back to k follow from those per position.
//
// The chunk-aware trim (a variant the pages leave open) first drops whole runs of the union
// that hold no anchor, weakest first by their best score (ties: the later run), while a whole
// run fits in the excess; the token-level trim then takes the rest.
//
// Threads own contiguous chunks of positions, so every scan is one in-chunk pass plus one
// block-level exclusive scan of chunk aggregates. Every function here is block-collective
// over kSelThreads threads.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace kara {

namespace {

constexpr int kSelThreads = 256;
constexpr int kWarps = kSelThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 sorts with +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan over thread index (forward: lower threads first; backward: higher first).
template <bool kForward, typename T, typename Op>
__device__ T block_exclusive_scan(T v, T identity, Op op, T* warp_buf) {
  const int lane = lane_id(), warp = warp_id();
  T x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    T y = kForward ? __shfl_up_sync(0xffffffffu, x, off) : __shfl_down_sync(0xffffffffu, x, off);
    if (kForward ? (lane >= off) : (lane + off < 32)) x = op(x, y);
  }
  // x: inclusive scan within the warp (in scan direction)
  T excl_in_warp = kForward ? __shfl_up_sync(0xffffffffu, x, 1) : __shfl_down_sync(0xffffffffu, x, 1);
  if (kForward ? (lane == 0) : (lane == 31)) excl_in_warp = identity;
  if (kForward ? (lane == 31) : (lane == 0)) warp_buf[warp] = x;
  __syncthreads();
  T carry = identity;
  if (kForward) {
    for (int w = 0; w < warp; ++w) carry = op(carry, warp_buf[w]);
  } else {
    for (int w = kWarps - 1; w > warp; --w) carry = op(carry, warp_buf[w]);
  }
  __syncthreads();
  return op(carry, excl_in_warp);
}

__device__ __forceinline__ int op_add(int a, int b) { return a + b; }
__device__ __forceinline__ int op_max(int a, int b) { return a > b ? a : b; }
__device__ __forceinline__ int op_min(int a, int b) { return a < b ? a : b; }

struct SelectSmem {
  uint32_t hist[256];
  int ibuf[kWarps];
  int digit;
  int above;
};

// Bytes of token2chunk_row's base arrays (the chunk-aware trim's arrays follow them).
__host__ __device__ constexpr size_t t2c_base_bytes(int W) {
  return sizeof(SelectSmem) + static_cast<size_t>(W) * 14;
}

// Among positions with cand[j] != 0, sets flag[j] = 1 for the `count` largest keys (ties:
// lower position first). Requires count <= number of candidates. Block-collective.
__device__ void block_select(const uint32_t* key, const uint8_t* cand, uint8_t* flag, int W,
                             int E, int count, SelectSmem* ss) {
  if (count <= 0) return;
  const int tid = threadIdx.x;
  const int lo = tid * E, hi = min(W, lo + E);
  uint32_t prefix = 0, mask = 0;
  int remaining = count;
  for (int shift = 24; shift >= 0; shift -= 8) {
    ss->hist[tid] = 0;
    __syncthreads();
    for (int j = lo; j < hi; ++j) {
      const uint32_t kj = key[j];
      if (cand[j] && (kj & mask) == prefix) atomicAdd(&ss->hist[(kj >> shift) & 255u], 1u);
    }
    __syncthreads();
    // thread tid looks at digit 255 - tid; counts of larger digits come first
    const int c = static_cast<int>(ss->hist[255 - tid]);
    const int before = block_exclusive_scan<true>(c, 0, op_add, ss->ibuf);
    if (before < remaining && remaining <= before + c) {
      ss->digit = 255 - tid;
      ss->above = before;
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(ss->digit) << shift;
    mask |= 0xffu << shift;
    remaining -= ss->above;
    __syncthreads();
  }
  // prefix = T, the count-th largest key; take everything above it and the first
  // `remaining` positions equal to it.
  int eq = 0;
  for (int j = lo; j < hi; ++j)
    if (cand[j] && key[j] == prefix) ++eq;
  int rank = block_exclusive_scan<true>(eq, 0, op_add, ss->ibuf);
  for (int j = lo; j < hi; ++j) {
    if (!cand[j]) continue;
    const uint32_t kj = key[j];
    if (kj > prefix) {
      flag[j] = 1;
    } else if (kj == prefix) {
      if (rank < remaining) flag[j] = 1;
      ++rank;
    }
  }
  __syncthreads();
}

// Writes the flagged positions of [0, W) in ascending order to out[0..].
__device__ void block_compact_write(const uint8_t* flag, int W, int E, int32_t* out,
                                    int* warp_buf) {
  const int lo = threadIdx.x * E, hi = min(W, lo + E);
  int cnt = 0;
  for (int j = lo; j < hi; ++j) cnt += flag[j];
  int pos = block_exclusive_scan<true>(cnt, 0, op_add, warp_buf);
  for (int j = lo; j < hi; ++j)
    if (flag[j]) out[pos++] = j;
}

// Chunk-aware trim, before the token-level trim: the runs of U that hold no anchor (all their
// members have priority 0) are dropped whole, weakest first by their best key (ties: the later
// run first), while the whole run fits in the excess |U| - k; their members get priority -1.
// run_s[j] is the start of the run of U around member j. Work arrays (in `cs`, chunk_smem(W)
// bytes): rkey / rlen / rrank per run start, the run starts listed ascending, the lengths by
// rank. Ranks are counted pairwise (O(R^2) for R unanchored runs, R <= k).
__device__ void drop_weak_runs(const uint32_t* key, const uint8_t* in_u, int8_t* prio,
                               const int16_t* run_s, int W, int E, int k, SelectSmem* ss,
                               uint8_t* cs) {
  uint32_t* rkey = reinterpret_cast<uint32_t*>(cs);
  int* rlen = reinterpret_cast<int*>(rkey + W);
  int* rrank = rlen + W;
  int* bylen = rrank + W;
  int16_t* list = reinterpret_cast<int16_t*>(bylen + W);
  __shared__ int s_total, s_runs, s_drop;
  const int tid = threadIdx.x;
  const int lo = tid * E, hi = min(W, lo + E);
  for (int j = tid; j < W; j += kSelThreads) {
    rkey[j] = 0u;
    rlen[j] = 0;
  }
  __syncthreads();
  int members = 0, starts = 0;
  for (int j = lo; j < hi; ++j) {
    if (!in_u[j]) continue;
    ++members;
    if (prio[j] != 0) continue;
    atomicMax(&rkey[run_s[j]], key[j]);
    atomicAdd(&rlen[run_s[j]], 1);
    if (run_s[j] == j) ++starts;
  }
  const int mem_before = block_exclusive_scan<true>(members, 0, op_add, ss->ibuf);
  int pos = block_exclusive_scan<true>(starts, 0, op_add, ss->ibuf);
  if (tid == kSelThreads - 1) {
    s_total = mem_before + members;
    s_runs = pos + starts;
  }
  for (int j = lo; j < hi; ++j)
    if (in_u[j] && prio[j] == 0 && run_s[j] == j) list[pos++] = static_cast<int16_t>(j);
  __syncthreads();
  const int R = s_runs, excess = s_total - k;
  // rank of each run: the number of weaker runs (smaller best key, or equal and later start)
  for (int r = tid; r < R; r += kSelThreads) {
    const int sr = list[r];
    const uint32_t kr = rkey[sr];
    int rank = 0;
    for (int q = 0; q < R; ++q) {
      const int sq = list[q];
      const uint32_t kq = rkey[sq];
      rank += (kq < kr || (kq == kr && sq > sr)) ? 1 : 0;
    }
    rrank[sr] = rank;
    bylen[rank] = rlen[sr];
  }
  __syncthreads();
  // the weakest runs whose lengths add up to at most the excess: ranks [0, s_drop)
  const int ER = (R + kSelThreads - 1) / kSelThreads;
  const int rlo = tid * ER, rhi = min(R, rlo + ER);
  int sum = 0;
  for (int r = rlo; r < rhi; ++r) sum += bylen[r];
  int acc = block_exclusive_scan<true>(sum, 0, op_add, ss->ibuf);
  int fits = 0;
  for (int r = rlo; r < rhi; ++r) {
    acc += bylen[r];
    if (acc <= excess) ++fits;
  }
  const int fits_before = block_exclusive_scan<true>(fits, 0, op_add, ss->ibuf);
  if (tid == kSelThreads - 1) s_drop = fits_before + fits;
  __syncthreads();
  const int ndrop = s_drop;
  for (int j = lo; j < hi; ++j)
    if (in_u[j] && prio[j] == 0 && rrank[run_s[j]] < ndrop) prio[j] = -1;
  __syncthreads();
}

// Token2Chunk of one row (block-level): s = the row's W scores, keep = where its k kept
// positions go (global or shared memory). The selection comes from sel_in (k positions), or,
// when sel_in is null, is selected here first (written to sel_out unless that is null).
// trim: KARA_TRIM_TOKEN, or KARA_TRIM_CHUNK (whole unanchored runs dropped first).
// smem: t2c_smem(W) bytes of shared memory, plus chunk_smem(W) more for the chunk-aware trim,
// 16-byte aligned.
__device__ void token2chunk_row(const float* __restrict__ s, const int32_t* sel_in,
                                int32_t* sel_out, int W, int k, int num_anchors, int gap_limit,
                                int widen, int32_t* keep, uint8_t* smem,
                                int trim = KARA_TRIM_TOKEN) {
  const bool kSelIn = sel_in != nullptr;
  SelectSmem* ss = reinterpret_cast<SelectSmem*>(smem);
  uint32_t* key = reinterpret_cast<uint32_t*>(smem + sizeof(SelectSmem));
  int16_t* prev_a = reinterpret_cast<int16_t*>(key + W);   // max anchor <= p, or -1
  int16_t* next_a = prev_a + W;                           // min anchor >= p, or W
  uint8_t* in_sel = reinterpret_cast<uint8_t*>(next_a + W);
  uint8_t* anchor = in_sel + W;
  uint8_t* in_u = anchor + W;
  int8_t* prio = reinterpret_cast<int8_t*>(in_u + W);
  uint8_t* cand = reinterpret_cast<uint8_t*>(prio + W);
  uint8_t* flag = cand + W;
  // chunk-aware trim only: the start of each member's run, then the work arrays
  int16_t* run_s = reinterpret_cast<int16_t*>(smem + ((t2c_base_bytes(W) + 15) / 16) * 16);
  uint8_t* chunk_ws = reinterpret_cast<uint8_t*>(run_s) + ((2 * W + 15) / 16) * 16;

  const int32_t* sl = sel_in;
  const int tid = threadIdx.x;
  const int E = (W + kSelThreads - 1) / kSelThreads;
  const int lo = tid * E, hi = min(W, lo + E);

  for (int j = tid; j < W; j += kSelThreads) {
    key[j] = order_key(s[j]);
    in_sel[j] = 0;
    anchor[j] = 0;
    flag[j] = 0;
    if (!kSelIn) cand[j] = 1;
  }
  __syncthreads();
  if (kSelIn) {
    for (int i = tid; i < k; i += kSelThreads) {
      const int p = sl[i];
      if (p >= 0 && p < W) in_sel[p] = 1;
    }
    __syncthreads();
  } else {
    // the selection itself: the k largest scores (ties: lower position) into in_sel
    block_select(key, cand, in_sel, W, E, k, ss);
    if (sel_out != nullptr) block_compact_write(in_sel, W, E, sel_out, ss->ibuf);
    __syncthreads();
  }

  // a. anchors: top num_anchors of the selection
  block_select(key, in_sel, anchor, W, E, num_anchors, ss);

  // previous / next anchor (inclusive)
  int cmax = -1, cmin = W;
  for (int j = lo; j < hi; ++j)
    if (anchor[j]) { cmax = j; if (cmin == W) cmin = j; }
  int carry_prev = block_exclusive_scan<true>(cmax, -1, op_max, ss->ibuf);
  int carry_next = block_exclusive_scan<false>(cmin, W, op_min, ss->ibuf);
  {
    int run = carry_prev;
    for (int j = lo; j < hi; ++j) {
      if (anchor[j]) run = j;
      prev_a[j] = static_cast<int16_t>(run);
    }
    run = carry_next;
    for (int j = hi - 1; j >= lo; --j) {
      if (anchor[j]) run = j;
      next_a[j] = static_cast<int16_t>(run);
    }
  }
  // b-d. gap fill, widen, union
  for (int j = lo; j < hi; ++j) {
    const int a = prev_a[j], b = next_a[j];
    bool u = in_sel[j] || anchor[j];
    if (!anchor[j] && a >= 0 && b < W && (b - a - 1) <= gap_limit) u = true;   // fill
    if (a >= 0 && j - a <= widen) u = true;                                     // widen
    if (b < W && b - j <= widen) u = true;
    in_u[j] = u ? 1 : 0;
  }
  __syncthreads();
  // previous / next non-member (inclusive) -> runs of U
  cmax = -1;
  cmin = W;
  for (int j = lo; j < hi; ++j)
    if (!in_u[j]) { cmax = j; if (cmin == W) cmin = j; }
  const int carry_gap_prev = block_exclusive_scan<true>(cmax, -1, op_max, ss->ibuf);
  const int carry_gap_next = block_exclusive_scan<false>(cmin, W, op_min, ss->ibuf);
  // e. priorities. The run of U around j is [last_gap+1, next_gap-1]; it holds an anchor iff
  // the nearest anchor on the left (prev_a) or on the right (next_a) falls inside it.
  {
    int last_gap = carry_gap_prev;
    for (int j = lo; j < hi; ++j) {
      if (!in_u[j]) last_gap = j;
      if (anchor[j]) prio[j] = 2;
      else if (in_u[j]) prio[j] = (prev_a[j] > last_gap) ? 1 : 0;
      else prio[j] = -1;
      if (trim == KARA_TRIM_CHUNK) run_s[j] = static_cast<int16_t>(last_gap + 1);
    }
    int next_gap = carry_gap_next;
    for (int j = hi - 1; j >= lo; --j) {
      if (!in_u[j]) next_gap = j;
      if (prio[j] == 0 && next_a[j] < next_gap) prio[j] = 1;
    }
  }
  __syncthreads();
  if (trim == KARA_TRIM_CHUNK) drop_weak_runs(key, in_u, prio, run_s, W, E, k, ss, chunk_ws);

  // f. trim to k by (priority, score, -position)
  int c1 = 0;
  for (int j = lo; j < hi; ++j) {
    if (prio[j] == 2) flag[j] = 1;
    c1 += (prio[j] == 1);
  }
  __shared__ int c1_sum;
  const int c1_before = block_exclusive_scan<true>(c1, 0, op_add, ss->ibuf);
  if (tid == kSelThreads - 1) c1_sum = c1_before + c1;
  __syncthreads();
  const int c2 = num_anchors;
  const int need1 = min(c1_sum, k - c2);
  for (int j = lo; j < hi; ++j) cand[j] = (prio[j] == 1);
  __syncthreads();
  block_select(key, cand, flag, W, E, need1, ss);
  const int need0 = k - c2 - need1;
  if (need0 > 0) {
    for (int j = lo; j < hi; ++j) cand[j] = (prio[j] == 0);
    __syncthreads();
    block_select(key, cand, flag, W, E, need0, ss);
  }
  block_compact_write(flag, W, E, keep, ss->ibuf);
}


__host__ __device__ constexpr size_t select_smem(int W) {
  return sizeof(SelectSmem) + static_cast<size_t>(W) * 6 + 64;
}
__host__ __device__ constexpr size_t t2c_smem(int W) {
  return sizeof(SelectSmem) + static_cast<size_t>(W) * 14 + 64;
}
// The chunk-aware trim's extra shared memory: run starts (int16) and five W-long work arrays.
__host__ __device__ constexpr size_t chunk_smem(int W) {
  return (static_cast<size_t>(2 * W) + 15) / 16 * 16 + static_cast<size_t>(W) * 18 + 64;
}

}  // namespace

}  // namespace kara
