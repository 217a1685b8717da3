// Window scoring on tcgen05 tensor cores (sm_100a).
//
// Computes, per due sequence r and KV head g,
//   score[j] = sum over the G query heads h of g and the window queries i of
//              softmax_j(q_hi . k_j * scale),
// bidirectional (unmasked) attention inside the compression window, column-summed
// ("Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression", English
// abstract: bidirectional attention scores the KV pairs of the window; gist.science explainer,
// section 1: a token the current reasoning refers to strongly scores high).
//
// Two passes, both persistent and warp-specialised (warp 0: TMA producer, warp 1: UMMA
// issuer and TMEM owner, the other warps: epilogue, one TMEM lane per thread, kParts warps per
// lane quadrant, each on 256/kParts of the accumulator columns):
//   pass 1 (query-major)  S = Q K^T, 128 query rows x up to 256 keys per UMMA tile; each
//                         epilogue thread owns one query row and keeps an online base-2
//                         log-sum-exp; the result goes to the workspace.
//   pass 2 (key-major)    S^T = K Q^T, 128 keys x 256 queries per tile; each epilogue thread
//                         owns one key and sums 2^(s*scale*log2e - lse_i) over all queries.
// Keys are read in place from the paged pool: a key tile is a run of whole 16-slot pages
// (TMA box of one page and one KV head); slots outside [n-W, n) are masked in the epilogue.
// Queries come from the dense window-query buffer [R, W, Hq, d]; rows past W are zero-filled
// by TMA and carry lse = +inf, so they add nothing in pass 2.
// The epilogues are bound by exponentials: a quarter of them run on the FMA pipe (ex2_fma2)
// and the rest on the SFU, so that both pipes share the load; the arithmetic around them
// uses packed fp32 pairs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>

#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace kara {

namespace {

constexpr int kEpiWarps = 8;                     // a multiple of 4: warps per TMEM lane quadrant
constexpr int kParts = kEpiWarps / 4;            // column parts of each 256-column accumulator
constexpr int kThreads = 64 + 32 * kEpiWarps;    // warp 0: TMA, warp 1: UMMA + TMEM, rest: epilogue
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kPartCols = 256 / kParts;          // accumulator columns per epilogue warp and tile
constexpr uint32_t kEpiBarrier = 1;  // named barrier among the epilogue warps
constexpr int kQRows1 = 128;         // pass 1: query rows per tile (UMMA M)
constexpr int kKRows1 = 256;         // pass 1: max keys per UMMA (N)
constexpr int kQStages1 = 2;
constexpr int kKRows2 = 128;         // pass 2: keys per tile (UMMA M)
constexpr int kQRows2 = 256;         // pass 2: queries per UMMA (N)
constexpr int kQStages2 = 2;
constexpr int kRowBytes = 128;       // one 64-element bf16 K-chunk row (128-byte swizzle)
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 accumulators

// Exponentials of 8 consecutive columns as 4 pairs: three pairs on the SFU, one pair on the
// FMA pipe (ex2_fma2). With the packed FFMA/FADD around them this balances issue slots
// against SFU cycles (the SFU delivers a quarter of a warp instruction per cycle per
// sub-partition).
__device__ __forceinline__ float2 exp2_pair(float2 x, int pair_in_group) {
  if (pair_in_group == 3) return ex2_fma2(x);
  return make_float2(ex2(x.x), ex2(x.y));
}

struct ScoreArgs {
  const int32_t* block_table;
  const int32_t* ctx_len;
  const int32_t* seq_ids;
  float* lse;         // [R, Hq, CM, Wp] base-2 log-sum-exp of scaled logits per query and
                      // key chunk (16 pages), from pass 1
  float* lse_merged;  // [R, Hq, Wp] the chunks merged (+inf past the window)
  int CM;             // key chunks per window, at most
  float* scores;    // [R, Hkv, W]
  float* part;      // fused kernel, split items: [split - 1][head part, tail part][W] key sums
  int streamk;      // fused kernel: cluster ranges split items (else they hold whole items)
  int ring;         // queries from the window-query ring [batch, 2W, Hq, d] (else q_win)
  float out_scale;  // 1, or 1 / (G W) for the mean aggregation
  int max_agg;      // the max aggregation (split parts combine by max)
  // A launch may cover part of the work: due rows [row0, row0 + R) (seq_ids and the query
  // rows are indexed by the global row; scores and the workspace by the local one, their
  // pointers starting at the range) and KV heads [g0, g0 + HkvN) of each (every head is
  // indexed globally); the fused kernel takes the first `items` (row, KV head) items.
  int row0, g0, HkvN;
  long long items;
  // The fused kernel with a helper beside it (a one-CTA-per-item two-pass kernel on the SMs
  // the clusters leave idle): each fused CTA adds 1 to *done_count when it leaves; CTA 0 of
  // the helper waits for done_target of them, so that what follows sees both kernels' work.
  int* done_count;
  int done_target;
  int32_t* status;
  int R, W, Wp, Hq, Hkv, G;
  int batch, max_blocks, num_blocks;
  float cs;         // scale * log2(e)
};

struct SeqInfo {
  int b, n, start, p_first, np;  // np: pages spanned by the window
  bool ok;
};

__device__ __forceinline__ SeqInfo seq_info(const ScoreArgs& a, int r) {
  SeqInfo s;
  s.b = a.seq_ids ? a.seq_ids[a.row0 + r] : a.row0 + r;
  s.ok = s.b >= 0 && s.b < a.batch;
  s.n = s.ok ? a.ctx_len[s.b] : 0;
  s.ok = s.ok && s.n >= a.W && s.n <= a.max_blocks * 16;
  s.start = s.n - a.W;
  s.p_first = s.ok ? s.start / 16 : 0;
  s.np = s.ok ? (s.n - 1) / 16 - s.p_first + 1 : 0;
  return s;
}

// Row and batch coordinates of the query tile that starts at window position row0: in the
// dense q_win [R, W, Hq, d] (due sequence r), or in the window-query ring [batch, 2W, Hq, d]
// (cache row b; window position 0 is ring row (n - W) mod W, and the W rows from there are
// contiguous because every query is stored at rows s mod W and s mod W + W).
__device__ __forceinline__ int q_tile_row(const ScoreArgs& a, const SeqInfo& s, int row0) {
  return a.ring ? s.start % a.W + row0 : row0;
}
__device__ __forceinline__ int q_tile_batch(const ScoreArgs& a, const SeqInfo& s, int r) {
  return a.ring ? s.b : a.row0 + r;
}

// Block id of page p of sequence row b, with range check (an out-of-range id is reported and
// replaced by block 0 so that the pipeline keeps its byte counts and never stalls).
__device__ __forceinline__ int page_block(const ScoreArgs& a, int b, int p) {
  int blk = a.block_table[static_cast<size_t>(b) * a.max_blocks + p];
  if (blk < 0 || blk >= a.num_blocks) {
    report(a.status, KARA_ERR_BAD_BLOCK);
    blk = 0;
  }
  return blk;
}

// Pass-2 work list: tiles (r, g, kt) in (r, g)-major order, ceil(np/8) key tiles per valid
// sequence (8 pages of 16 keys each) and ceil(W/128) zero-writing tiles per invalid one. Every
// role of a CTA walks it with its own cursor; the tile index only grows, so the cursor only
// moves forward.
struct TileCursor {
  int r = 0, base = 0, per = -1;
  SeqInfo s;
  __device__ __forceinline__ bool seek(const ScoreArgs& a, int t, int& g, int& kt) {
    while (true) {
      if (r >= a.R) return false;
      if (per < 0) {
        s = seq_info(a, r);
        per = s.ok ? (s.np + 7) / 8 : (a.W + kKRows2 - 1) / kKRows2;
      }
      if (t < base + a.HkvN * per) break;
      base += a.HkvN * per;
      ++r;
      per = -1;
    }
    const int local = t - base;
    g = a.g0 + local / per;
    kt = local % per;
    return true;
  }
};

// Pass-1 work list: tiles (r, g, c, hl) = key chunk c (16 pages of KV head g) against the
// window queries of query head g*G + hl, for valid sequences only, (r, g, c)-major so that
// neighbouring tiles share the key chunk in L2.
struct RowTileCursor {
  int r = 0, base = 0, per = -1, nc = 0;
  SeqInfo s;
  __device__ __forceinline__ bool seek(const ScoreArgs& a, int t, int& g, int& c, int& hl) {
    while (true) {
      if (r >= a.R) return false;
      if (per < 0) {
        s = seq_info(a, r);
        nc = s.ok ? (s.np + 15) / 16 : 0;
        per = a.HkvN * nc * a.G;
      }
      if (t < base + per) break;
      base += per;
      ++r;
      per = -1;
    }
    int local = t - base;
    hl = local % a.G;
    local /= a.G;
    c = local % nc;
    g = a.g0 + local / nc;
    return true;
  }
};

// ----------------------------------------------------------------------------------------
// Pass 1: per-query base-2 log-sum-exp over each 16-page key chunk of the window.
// The chunk (up to 256 keys) stays in shared memory while 128-query tiles of one query head
// stream through it: S = Q K^T (UMMA M = 128 queries, N = the chunk's keys). The partial
// results of the chunks are merged when pass 2 stages them.
// ----------------------------------------------------------------------------------------
// The pass as a device function over the tiles t0, t0 + tstep, ... of the cursor (a kernel
// passes its CTA index and the grid size; the one-CTA item kernel 0 and 1), on the
// 1024-aligned shared memory `smem`. `relinquish`: release the CTA's right to allocate
// tensor memory after this pass's allocation (the item kernel allocates again).
template <int D>
__device__ __forceinline__ void rowstats_pass(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                              const ScoreArgs& a, uint8_t* smem, int t0,
                                              int tstep, bool relinquish) {
  constexpr int NCH = D / 64;
  constexpr uint32_t kQBytes = NCH * kQRows1 * kRowBytes;
  constexpr uint32_t kKBytes = NCH * kKRows1 * kRowBytes;
  constexpr uint32_t kPageBytes = 16 * kRowBytes;
  uint8_t* k_buf = smem;                      // 2 x kKBytes (key chunks)
  uint8_t* q_buf = smem + 2 * kKBytes;        // kQStages1 x kQBytes (query tiles)
  float2* comb = reinterpret_cast<float2*>(q_buf + kQStages1 * kQBytes);   // [kParts-1][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(comb + 3 * kQRows1);
  uint64_t* k_full = bars;                    // [2]
  uint64_t* k_empty = bars + 2;               // [2]
  uint64_t* q_full = bars + 4;                // [kQStages1]
  uint64_t* q_empty = bars + 4 + kQStages1;
  uint64_t* acc_full = bars + 4 + 2 * kQStages1;   // [2]
  uint64_t* acc_empty = acc_full + 2;              // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int TT = (a.W + kQRows1 - 1) / kQRows1;   // query tiles per head

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads);
    }
    for (int i = 0; i < kQStages1; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    if (relinquish) tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---- TMA producer (whole warp: lanes fetch page ids, lane 0 issues the copies) ----
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
    }
    int ki = 0, qi = 0;
    uint32_t kph = 0, qph = 0;
    RowTileCursor cur;
    int g, c, hl;
    for (int t = t0; cur.seek(a, t, g, c, hl); t += tstep) {
      if (__shfl_sync(0xffffffffu, *abort_flag != 0 ? 1 : 0, 0)) break;
      const SeqInfo& s = cur.s;
      const int r = cur.r;
      const int h = g * a.G + hl;
      const int pages = min(16, s.np - c * 16);
      const int my_blk = lane < pages ? page_block(a, s.b, s.p_first + c * 16 + lane) : 0;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&k_empty[ki], kph ^ 1, abort_flag, a.status) ? 1 : 0;
        if (ok) mbar_expect_tx(&k_full[ki], pages * NCH * kPageBytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int p = 0; p < pages; ++p) {
        const int blk = __shfl_sync(0xffffffffu, my_blk, p);
        if (lane == 0) {
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_4d(k_buf + ki * kKBytes + ch * kKRows1 * kRowBytes + p * kPageBytes, &tm_k,
                        &k_full[ki], ch * 64, g, 0, blk);
        }
      }
      if (++ki == 2) { ki = 0; kph ^= 1; }
      bool stop = false;
      if (lane == 0) {
        for (int qt = 0; qt < TT; ++qt) {
          if (!mbar_wait(&q_empty[qi], qph ^ 1, abort_flag, a.status)) { stop = true; break; }
          mbar_expect_tx(&q_full[qi], kQBytes);
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_4d(q_buf + qi * kQBytes + ch * kQRows1 * kRowBytes, &tm_q, &q_full[qi],
                        ch * 64, h, q_tile_row(a, s, qt * kQRows1), q_tile_batch(a, s, r));
          if (++qi == kQStages1) { qi = 0; qph ^= 1; }
        }
      }
      qi = __shfl_sync(0xffffffffu, qi, 0);
      qph = __shfl_sync(0xffffffffu, qph, 0);
      if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) break;
    }
  } else if (warp == 1) {
    // ---------------- UMMA issuer ----------------
    if (lane == 0) {
      int ki = 0, qi = 0, ab = 0;
      uint32_t kph = 0, qph = 0, aph = 0;
      RowTileCursor cur;
      int g, c, hl;
      for (int t = t0; !*abort_flag && cur.seek(a, t, g, c, hl); t += tstep) {
        const SeqInfo& s = cur.s;
        const int pages = min(16, s.np - c * 16);
        if (!mbar_wait(&k_full[ki], kph, abort_flag, a.status)) break;
        const uint32_t k_addr = smem_u32(k_buf + ki * kKBytes);
        const uint32_t idesc = idesc_bf16_f32(128, pages * 16);
        bool stop = false;
        for (int qt = 0; qt < TT; ++qt) {
          if (!mbar_wait(&q_full[qi], qph, abort_flag, a.status)) { stop = true; break; }
          if (!mbar_wait(&acc_empty[ab], aph ^ 1, abort_flag, a.status)) { stop = true; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(q_buf + qi * kQBytes);
          const uint32_t d_tmem = tmem_base + ab * 256;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t ad = sw128_kmajor_desc(q_addr + (kk >> 2) * kQRows1 * kRowBytes + off);
            const uint64_t bd = sw128_kmajor_desc(k_addr + (kk >> 2) * kKRows1 * kRowBytes + off);
            umma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&q_empty[qi]);
          umma_commit(&acc_full[ab]);
          if (++qi == kQStages1) { qi = 0; qph ^= 1; }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        if (stop) break;
        umma_commit(&k_empty[ki]);
        if (++ki == 2) { ki = 0; kph ^= 1; }
      }
    }
  } else {
    // ------- epilogue: one query row per TMEM lane, kParts warps per lane quadrant -------
    const int e = warp - 2;
    const int quad = warp & 3;
    const int part = e >> 2;              // which kPartCols columns of each tile
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const float2 cs2 = make_float2(a.cs, a.cs);
    int ab = 0;
    uint32_t aph = 0;
    bool aborted = false;
    RowTileCursor cur;
    int g, c, hl;
    for (int t = t0; cur.seek(a, t, g, c, hl); t += tstep) {
      const SeqInfo& s = cur.s;
      const int r = cur.r;
      const int h = g * a.G + hl;
      const int nc = cur.nc;
      const int ncols = min(16, s.np - c * 16) * 16;
      const int c0 = part * kPartCols;
      const int cnt = max(0, min(kPartCols, ncols - c0));     // a multiple of 16
      const int nch = (cnt + 31) / 32;
      const int slot0 = (s.p_first + c * 16) * 16 + c0;
      const bool edge = (c == 0) || (c == nc - 1);
      float* lrow = a.lse + ((static_cast<size_t>(r) * a.Hq + h) * a.CM + c) * a.Wp;
      for (int qt = 0; qt < TT; ++qt) {
        float m = -INFINITY, l = 0.f;
        if (!aborted && !mbar_wait(&acc_full[ab], aph, abort_flag, a.status)) aborted = true;
        if (!aborted) {
          tc_fence_after();
          const uint32_t col0 = lane_base + ab * 256 + c0;
          // one 32-column chunk: masked max, rescale, exponentials
          auto process = [&](float (&v)[32], int j) {
            if (cnt - 32 * j == 16) {
#pragma unroll
              for (int i = 16; i < 32; ++i) v[i] = -INFINITY;
            }
            if (edge) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int slot = slot0 + 32 * j + i;
                if (slot < s.start || slot >= s.n) v[i] = -INFINITY;
              }
            }
            float mx[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float a0 = fmaxf(v[8 * q], v[8 * q + 1]), a1 = fmaxf(v[8 * q + 2], v[8 * q + 3]);
              const float a2 = fmaxf(v[8 * q + 4], v[8 * q + 5]), a3 = fmaxf(v[8 * q + 6], v[8 * q + 7]);
              mx[q] = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
            }
            const float cmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (cmax == -INFINITY) return;
            const float m_new = fmaxf(m, cmax * a.cs);
            const float2 nm2 = make_float2(-m_new, -m_new);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float2 x0 = ffma2(make_float2(v[i], v[i + 1]), cs2, nm2);
              const float2 x1 = ffma2(make_float2(v[i + 2], v[i + 3]), cs2, nm2);
              acc0 = fadd2(acc0, exp2_pair(x0, (i >> 1) & 3));
              acc1 = fadd2(acc1, exp2_pair(x1, ((i >> 1) + 1) & 3));
            }
            const float2 acc = fadd2(acc0, acc1);
            l = l * ex2(m - m_new) + (acc.x + acc.y);
            m = m_new;
          };
          auto issue = [&](float (&v)[32], int j) {
            tmem_ld16(col0 + 32 * j, v);
            if (cnt - 32 * j > 16) tmem_ld16(col0 + 32 * j + 16, v + 16);
          };
          float va[32], vb[32];
          if (nch > 0) issue(va, 0);
          for (int j = 0; j < nch; j += 2) {
            tmem_wait_ld();
            reg_fence<32>(va);
            if (j + 1 < nch) issue(vb, j + 1);
            if (j + 1 >= nch) {            // all of this part's columns are in registers
              tc_fence_before();
              mbar_arrive(&acc_empty[ab]);
            }
            process(va, j);
            if (j + 1 < nch) {
              tmem_wait_ld();
              reg_fence<32>(vb);
              if (j + 2 < nch) issue(va, j + 2);
              else {
                tc_fence_before();
                mbar_arrive(&acc_empty[ab]);
              }
              process(vb, j + 1);
            }
          }
          if (nch == 0) {
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);
          }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        // merge the column parts of the row; part 0 writes the chunk's partial lse
        if (part > 0) comb[(part - 1) * kQRows1 + row] = make_float2(m, l);
        named_barrier(kEpiBarrier, kEpiThreads);
        if (part == 0) {
          float mm = m;
          float2 o[kParts - 1];
#pragma unroll
          for (int q = 0; q < kParts - 1; ++q) {
            o[q] = comb[q * kQRows1 + row];
            mm = fmaxf(mm, o[q].x);
          }
          float ll = (m == -INFINITY) ? 0.f : l * ex2(m - mm);
#pragma unroll
          for (int q = 0; q < kParts - 1; ++q)
            if (o[q].x != -INFINITY) ll += o[q].y * ex2(o[q].x - mm);
          const int token = qt * kQRows1 + row;
          if (token < a.Wp) lrow[token] = (aborted || ll == 0.f) ? -INFINITY : mm + __log2f(ll);
        }
        named_barrier(kEpiBarrier, kEpiThreads);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {   // the barriers' memory may be reused by a later pass
    for (int i = 0; i < 4 + 2 * kQStages1 + 4; ++i) mbar_inval(&bars[i]);
  }
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_rowstats_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  rowstats_pass<D>(tm_q, tm_k, a, smem, blockIdx.x, gridDim.x, true);
}


// ----------------------------------------------------------------------------------------
// Merge of the per-chunk partial log-sum-exps: lse = log2(sum_c 2^lse_c), one thread per query.
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) score_lse_merge_kernel(const ScoreArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  const size_t total = static_cast<size_t>(a.R) * a.Hq * a.Wp;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int token = static_cast<int>(i % a.Wp);
    const size_t rh = i / a.Wp;
    const int r = static_cast<int>(rh / a.Hq);
    float out = INFINITY;
    if (token < a.W) {
      const SeqInfo s = seq_info(a, r);
      if (s.ok) {
        const int nc = (s.np + 15) / 16;
        const float* p = a.lse + rh * a.CM * a.Wp + token;
        float mx = -INFINITY;
        for (int c = 0; c < nc; ++c) mx = fmaxf(mx, p[static_cast<size_t>(c) * a.Wp]);
        float sum = 0.f;
        for (int c = 0; c < nc; ++c) sum += ex2(p[static_cast<size_t>(c) * a.Wp] - mx);
        out = mx + __log2f(sum);
      }
    }
    a.lse_merged[i] = out;
  }
}

// ----------------------------------------------------------------------------------------
// Pass 2: per-key sums of the normalised probabilities.
// ----------------------------------------------------------------------------------------
// kMax: the largest probability of each key over the group's queries in place of the sum:
// max_i 2^(s c - lse_i) = 2^(max_i (s c - lse_i)), one exponential per key.
// The pass as a device function, as rowstats_pass.
template <int D, bool kMax>
__device__ __forceinline__ void colsum_pass(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                            const ScoreArgs& a, uint8_t* smem, int t0,
                                            int tstep, bool relinquish) {
  constexpr int NCH = D / 64;
  constexpr uint32_t kABytes = NCH * kKRows2 * kRowBytes;
  constexpr uint32_t kBBytes = NCH * kQRows2 * kRowBytes;
  constexpr uint32_t kPageBytes = 16 * kRowBytes;
  uint8_t* a_buf = smem;                    // 2 x kABytes (key tiles)
  uint8_t* b_buf = smem + 2 * kABytes;      // kQStages2 x kBBytes (query tiles)
  float* lse_s = reinterpret_cast<float*>(b_buf + kQStages2 * kBBytes);   // [2][256]
  float* red = lse_s + 2 * kQRows2;                                       // [3][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 3 * kKRows2);
  uint64_t* a_full = bars;                  // [2]
  uint64_t* a_empty = bars + 2;             // [2]
  uint64_t* b_full = bars + 4;              // [kQStages2]
  uint64_t* b_empty = bars + 4 + kQStages2;
  uint64_t* acc_full = bars + 4 + 2 * kQStages2;   // [2]
  uint64_t* acc_empty = acc_full + 2;              // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int QT = (a.W + kQRows2 - 1) / kQRows2;
  const int NQ = a.G * QT;                  // query tiles per key tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads);
    }
    for (int i = 0; i < kQStages2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    if (relinquish) tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // whole warp: lanes fetch the tile's page ids in parallel, lane 0 issues the copies
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
    }
    int ai = 0, bi = 0;
    uint32_t aph = 0, bph = 0;
    TileCursor cur;
    int g, kt;
    for (int t = t0; cur.seek(a, t, g, kt); t += tstep) {
      if (__shfl_sync(0xffffffffu, *abort_flag != 0 ? 1 : 0, 0)) break;
      const SeqInfo& s = cur.s;
      if (!s.ok) continue;
      const int r = cur.r;
      const int pages = min(8, s.np - kt * 8);
      const int my_blk = lane < pages ? page_block(a, s.b, s.p_first + kt * 8 + lane) : 0;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&a_empty[ai], aph ^ 1, abort_flag, a.status) ? 1 : 0;
        if (ok) mbar_expect_tx(&a_full[ai], pages * NCH * kPageBytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int p = 0; p < pages; ++p) {
        const int blk = __shfl_sync(0xffffffffu, my_blk, p);
        if (lane == 0) {
          for (int c = 0; c < NCH; ++c)
            tma_load_4d(a_buf + ai * kABytes + c * kKRows2 * kRowBytes + p * kPageBytes, &tm_k,
                        &a_full[ai], c * 64, g, 0, blk);
        }
      }
      if (++ai == 2) { ai = 0; aph ^= 1; }
      bool stop = false;
      if (lane == 0) {
        for (int q = 0; q < NQ; ++q) {
          const int h = g * a.G + q / QT, qt = q % QT;
          if (!mbar_wait(&b_empty[bi], bph ^ 1, abort_flag, a.status)) { stop = true; break; }
          mbar_expect_tx(&b_full[bi], kBBytes);
          for (int c = 0; c < NCH; ++c)
            tma_load_4d(b_buf + bi * kBBytes + c * kQRows2 * kRowBytes, &tm_q, &b_full[bi],
                        c * 64, h, q_tile_row(a, s, qt * kQRows2), q_tile_batch(a, s, r));
          if (++bi == kQStages2) { bi = 0; bph ^= 1; }
        }
      }
      // lanes other than 0 track the stage index too (they only read it on the next tile)
      bi = __shfl_sync(0xffffffffu, bi, 0);
      bph = __shfl_sync(0xffffffffu, bph, 0);
      if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int ai = 0, bi = 0, ab = 0;
      uint32_t aph = 0, bph = 0, cph = 0;
      const uint32_t idesc = idesc_bf16_f32(128, kQRows2);
      TileCursor cur;
      int g, kt;
      for (int t = t0; !*abort_flag && cur.seek(a, t, g, kt); t += tstep) {
        if (!cur.s.ok) continue;
        if (!mbar_wait(&a_full[ai], aph, abort_flag, a.status)) break;
        const uint32_t a_addr = smem_u32(a_buf + ai * kABytes);
        bool stop = false;
        for (int q = 0; q < NQ; ++q) {
          if (!mbar_wait(&b_full[bi], bph, abort_flag, a.status)) { stop = true; break; }
          if (!mbar_wait(&acc_empty[ab], cph ^ 1, abort_flag, a.status)) { stop = true; break; }
          tc_fence_after();
          const uint32_t b_addr = smem_u32(b_buf + bi * kBBytes);
          const uint32_t d_tmem = tmem_base + ab * 256;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t ad = sw128_kmajor_desc(a_addr + (kk >> 2) * kKRows2 * kRowBytes + off);
            const uint64_t bd = sw128_kmajor_desc(b_addr + (kk >> 2) * kQRows2 * kRowBytes + off);
            umma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&b_empty[bi]);
          umma_commit(&acc_full[ab]);
          if (++bi == kQStages2) { bi = 0; bph ^= 1; }
          if (++ab == 2) { ab = 0; cph ^= 1; }
        }
        if (stop) break;
        umma_commit(&a_empty[ai]);
        if (++ai == 2) { ai = 0; aph ^= 1; }
      }
    }
  } else {
    // ------------- epilogue: one key per TMEM lane, four warps per lane quadrant -------------
    const int e = warp - 2;
    const int etid = e * 32 + lane;       // 0..511; the first 256 stage the tile's lse values
    const int quad = warp & 3;
    const int part = e >> 2;              // which 64 query columns of each tile
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const float2 cs2 = make_float2(a.cs, a.cs);
    int ab = 0, qbuf = 0;
    uint32_t cph = 0;
    bool aborted = false;
    TileCursor cur;
    int g, kt;
    for (int t = t0; cur.seek(a, t, g, kt); t += tstep) {
      const SeqInfo& s = cur.s;
      const int r = cur.r;
      float* out = a.scores + (static_cast<size_t>(r) * a.Hkv + g) * a.W;
      if (!s.ok) {
        const int j = kt * kKRows2 + row;
        if (part == 0 && j < a.W) out[j] = 0.f;
        if (kt == 0 && g == 0 && etid == 0) report(a.status, KARA_ERR_INVALID_ARG);
        continue;
      }
      const float init = kMax ? -INFINITY : 0.f;
      float2 acc0 = make_float2(init, init), acc1 = make_float2(init, init);
      // merged lse of the tile's 256 queries, staged negated; the next tile's is prefetched
      const float* lse_rows = a.lse_merged + (static_cast<size_t>(r) * a.Hq + g * a.G) * a.Wp;
      float lv = etid < kQRows2 ? lse_rows[etid] : 0.f;
      for (int q = 0; q < NQ; ++q) {
        float* ls = lse_s + qbuf * kQRows2;
        if (etid < kQRows2) {
          ls[etid] = -lv;
          if (q + 1 < NQ) {
            const int h1 = (q + 1) / QT, qt1 = (q + 1) % QT;
            lv = lse_rows[static_cast<size_t>(h1) * a.Wp + qt1 * kQRows2 + etid];
          }
        }
        named_barrier(kEpiBarrier, kEpiThreads);
        if (!aborted && !mbar_wait(&acc_full[ab], cph, abort_flag, a.status)) aborted = true;
        if (!aborted) {
          tc_fence_after();
          const uint32_t col0 = lane_base + ab * 256 + part * kPartCols;
          const float* lh = ls + part * kPartCols;
          constexpr int nch = kPartCols / 32;
          auto issue = [&](float (&v)[32], int j) {
            tmem_ld16(col0 + 32 * j, v);
            tmem_ld16(col0 + 32 * j + 16, v + 16);
          };
          auto process = [&](const float (&v)[32], int j) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 nl = *reinterpret_cast<const float4*>(lh + 32 * j + i);
              const float2 x0 = ffma2(make_float2(v[i], v[i + 1]), cs2, make_float2(nl.x, nl.y));
              const float2 x1 = ffma2(make_float2(v[i + 2], v[i + 3]), cs2, make_float2(nl.z, nl.w));
              if (kMax) {
                acc0 = make_float2(fmaxf(acc0.x, x0.x), fmaxf(acc0.y, x0.y));
                acc1 = make_float2(fmaxf(acc1.x, x1.x), fmaxf(acc1.y, x1.y));
              } else {
                acc0 = fadd2(acc0, exp2_pair(x0, (i >> 1) & 3));
                acc1 = fadd2(acc1, exp2_pair(x1, ((i >> 1) + 1) & 3));
              }
            }
          };
          float va[32], vb[32];
          issue(va, 0);
#pragma unroll
          for (int j = 0; j < nch; j += 2) {
            tmem_wait_ld();
            reg_fence<32>(va);
            if (j + 1 < nch) issue(vb, j + 1);
            else {
              tc_fence_before();
              mbar_arrive(&acc_empty[ab]);
            }
            process(va, j);
            if (j + 1 < nch) {
              tmem_wait_ld();
              reg_fence<32>(vb);
              if (j + 2 < nch) issue(va, j + 2);
              else {
                tc_fence_before();
                mbar_arrive(&acc_empty[ab]);
              }
              process(vb, j + 1);
            }
          }
          if (++ab == 2) { ab = 0; cph ^= 1; }
        }
        qbuf ^= 1;
      }
      // merge the query parts of each key
      const float total = kMax ? fmaxf(fmaxf(acc0.x, acc0.y), fmaxf(acc1.x, acc1.y))
                               : (acc0.x + acc1.x) + (acc0.y + acc1.y);
      if (part > 0) red[(part - 1) * kKRows2 + row] = total;
      named_barrier(kEpiBarrier, kEpiThreads);
      if (part == 0 && !aborted) {
        const int slot = (s.p_first + kt * 8) * 16 + row;
        const int j = slot - s.start;
        float sum = total;
#pragma unroll
        for (int q = 0; q < kParts - 1; ++q)
          sum = kMax ? fmaxf(sum, red[q * kKRows2 + row]) : sum + red[q * kKRows2 + row];
        if (row < min(8, s.np - kt * 8) * 16 && j >= 0 && j < a.W)
          out[j] = kMax ? exp2f(sum) : sum * a.out_scale;
      }
      named_barrier(kEpiBarrier, kEpiThreads);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {   // the barriers' memory may be reused by a later pass
    for (int i = 0; i < 4 + 2 * kQStages2 + 4; ++i) mbar_inval(&bars[i]);
  }
  __syncthreads();
}

template <int D, bool kMax>
__global__ void __launch_bounds__(kThreads, 1)
score_colsum_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  colsum_pass<D, kMax>(tm_q, tm_k, a, smem, blockIdx.x, gridDim.x, true);
}

// ----------------------------------------------------------------------------------------
// The helper beside the fused kernel: one CTA takes whole (row, KV head) items, items
// item0 + blockIdx.x, + gridDim.x, ..., through both passes of the two-pass path (the row
// log-sum-exps of the item's G query heads, their merge over the key chunks, the column
// sums), so that it needs nothing from other CTAs. Launched as the fused kernel's
// programmatic dependent once that kernel's CTAs all run, on the SMs its clusters leave idle;
// it reads only what was complete before the fused kernel started, so it does not wait at
// entry. CTA 0 waits at the end for every fused CTA (a.done_count), so that the kernels after
// this one see both kernels' scores. Workspace: one row's two-pass region per CTA.
// ----------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_item_kernel(const __grid_constant__ CUtensorMap tm_q1,
                  const __grid_constant__ CUtensorMap tm_q2,
                  const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a, long long item0,
                  long long nitems) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const size_t region = static_cast<size_t>(a.Hq) * (a.CM + 1) * a.Wp;   // floats per CTA
  float* ws = a.lse + blockIdx.x * region;
  for (long long it = blockIdx.x; it < nitems; it += gridDim.x) {
    const long long item = item0 + it;
    const int r = static_cast<int>(item / a.Hkv);
    const int g = static_cast<int>(item - static_cast<long long>(r) * a.Hkv);
    ScoreArgs b = a;
    b.R = 1;
    b.row0 = r;
    b.g0 = g;
    b.HkvN = 1;
    b.scores = a.scores + static_cast<size_t>(r) * a.Hkv * a.W;
    b.lse = ws;
    b.lse_merged = ws + static_cast<size_t>(a.Hq) * a.CM * a.Wp;
    rowstats_pass<D>(tm_q1, tm_k, b, smem, 0, 1, false);
    // merge of the key chunks' partial log-sum-exps, the item's G query heads
    const SeqInfo s = seq_info(b, 0);
    const int nc = s.ok ? (s.np + 15) / 16 : 0;
    for (int i = threadIdx.x; i < a.G * a.Wp; i += blockDim.x) {
      const int h = g * a.G + i / a.Wp;
      const int token = i % a.Wp;
      float out = INFINITY;
      if (s.ok && token < a.W) {
        const float* p = b.lse + static_cast<size_t>(h) * a.CM * a.Wp + token;
        float mx = -INFINITY;
        for (int c = 0; c < nc; ++c) mx = fmaxf(mx, p[static_cast<size_t>(c) * a.Wp]);
        float sum = 0.f;
        for (int c = 0; c < nc; ++c) sum += ex2(p[static_cast<size_t>(c) * a.Wp] - mx);
        out = mx + __log2f(sum);
      }
      b.lse_merged[static_cast<size_t>(h) * a.Wp + token] = out;
    }
    __syncthreads();
    colsum_pass<D, false>(tm_q2, tm_k, b, smem, 0, 1, false);
  }
  if (a.done_count != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    const long long t0 = clock64();
    while (ld_acquire_gpu(a.done_count) < a.done_target) {
      if (clock64() - t0 > kWaitBudgetCycles) {
        report(a.status, KARA_ERR_TIMEOUT);
        break;
      }
      __nanosleep(500);
    }
  }
}

// ----------------------------------------------------------------------------------------
// Fused scoring: one exponential per score, on a cluster of CL = ceil(W / 128) CTAs (W <= 1024,
// or W = 2048 on 16).
//
// Work items are (r, g): the G query heads of KV head g of a valid sequence r against the
// window keys of that KV head (G * ceil(W / 128) query tiles); all CTAs of a cluster take the
// same items, CTA `rank` owns the window keys [start + 128 rank, start + 128 rank + 128) that
// exist (a window that is not a multiple of 128 leaves the last CTA fewer; its other S columns
// are set to -inf in tensor memory, so that they count nowhere). Per 128-query tile each CTA
//   1. computes S = Q K^T over its keys (UMMA M = 128 queries, N = 128 keys). The 9 pages that
//      cover the 128 keys at any slot offset are loaded whole; the B operand starts at the
//      first owned key's row inside them (the 128-byte swizzle is a function of the shared
//      memory address, so a start at any row of a 1024-byte-aligned buffer reads the rows as
//      the TMA wrote them);
//   2. in the epilogue (4 warps, one per TMEM lane quadrant: a thread owns one query row and
//      the CTA's 128 keys) takes the row max m over its keys, P' = 2^(s*c - m + 15) and the
//      row sum l, and stores P' as fp16 in shared memory, MN-major (rows along K) for the next
//      product;
//   3. sends the row's partial log-sum-exp over its 128 keys, lse = m + log2(l), to every CTA
//      of the cluster (st.async into their shared memory, counted on their mbarrier);
//   4. once all CL partials of a row are in: M = max lse, L = sum 2^(lse - M), and the row
//      weight w = 2^(m - M + 15) / L (so that P' w = 2^15 softmax); w goes to fp16 as three B
//      columns (w1 + w2 + 2^-24 w3, exact to about 2^-36);
//   5. D (128 keys x 16) += P'^T W: the column sums of the tile's softmax rows on the tensor
//      cores (UMMA M = 128 keys, K = 128 queries, N = 16), accumulated over the item's tiles.
// Three teams of 4 epilogue warps take the tiles in turn, each with its own S accumulator in
// TMEM and its own P' and weight buffers, so that a team's wait for the cluster exchange and
// its weights overlap the other two teams' exponentials. After the item's last tile, D (times
// 2^-15) holds the per-key scores summed over the item's G heads.
// ----------------------------------------------------------------------------------------
constexpr int kFTeams = 3;                        // epilogue teams, tile T goes to team T mod 3
constexpr int kFEpiWarps = 4 * kFTeams;           // a team: one warp per TMEM lane quadrant
constexpr int kFTeamThreads = 128;                // a thread owns one query row of the tile
// warps 0-3: TMA producer, S issuer, column-sum issuer, and a spare, so that each of the four
// SM sub-partitions holds one such warp beside its four epilogue warps
constexpr int kFThreads = 128 + 32 * kFEpiWarps;
constexpr int kFEpiThreads = 32 * kFEpiWarps;
constexpr int kFKeys = 128;            // window keys owned per CTA
constexpr int kFKRows = 144;           // key rows loaded per CTA (9 pages)
constexpr int kFQRows = 128;           // queries per tile
// the helper beside the fused kernel (score_item_kernel): used from this many idle SMs; an
// item's cost per SM on the two-pass path against the fused kernel's (clusters of up to 8,
// clusters of 16), measured: step workload 1.04 against 0.42 ms; 8B-GQA 2.07 against 1.05
constexpr int kHelperMinSms = 8;
constexpr double kHelperCost = 2.5;
constexpr double kHelperCost16 = 2.0;
constexpr int kFMaxCluster = 16;      // W = 2048: a non-portable cluster of 16 CTAs
constexpr int kFPBufs = kFTeams;       // S, P' and weight buffers, tile T in buffer T mod 3
// query ring slots of one 64-channel chunk each: three, or two for a cluster of 16 (whose
// exchange records need the room)
__host__ __device__ constexpr int fq_slots(int CL) { return CL > 8 ? 2 : 3; }
// query tiles between a tile's L2 prefetch and its load; only a ring of two slots (a cluster
// of 16) gains from it, three slots already cover the load latency
__host__ __device__ constexpr int fq_ahead(int CL) { return fq_slots(CL) < 3 ? 2 : 0; }
constexpr int kFXStages = 6;           // exchange slots: a peer sends its record of tile T + 6
                                       // only after its weights of tile T + 3, which need this
                                       // CTA's record of tile T + 3, which the team of tile T
                                       // sends after it has read the partials of tile T
constexpr uint32_t kFSCols = kFKeys;  // TMEM column stride of the three S buffers: 0, 128, 256
constexpr uint32_t kFDCol = kFTeams * kFSCols;   // TMEM columns of the two D buffers: 384, 400

// Work items (r, g): KV head g of sequence r with all G of its query heads, TPI = G * CL query
// tiles (tile tq: head g * G + tq / CL, queries 128 (tq % CL) ..; rows past W weigh nothing).
// Cluster c of ncl takes
// a contiguous range of the sequence of (item, tile) pairs, items in order:
//  - streamk: tiles [c N / ncl, (c + 1) N / ncl) of N = R * Hkv * TPI, so every cluster has the
//    same share within a tile. A boundary inside an item splits it into a head part (ending
//    cluster c - 1's range) and a tail part (starting cluster c's); each writes its key sums
//    to its slot of split c and a second kernel adds the two. Ranges are at least TPI tiles
//    long, so an item holds at most one boundary;
//  - otherwise: whole items [c I / ncl, (c + 1) I / ncl) of I = R * Hkv.
// A segment is the range's part of one item, tiles [q0, q1); items of invalid sequences are
// skipped.
struct SegCursor {
  long long t = 0, t1 = 0;
  int r = 0, g = 0, q0 = 0, q1 = 0;
  SeqInfo s;
  __device__ __forceinline__ void init(const ScoreArgs& a, int c, int ncl, int TPI) {
    const long long items = a.items;
    if (a.streamk) {
      const long long n = items * TPI;
      t = c * n / ncl;
      t1 = (c + 1) * n / ncl;
    } else {
      t = c * items / ncl * TPI;
      t1 = (c + 1) * items / ncl * TPI;
    }
  }
  __device__ __forceinline__ bool next(const ScoreArgs& a, int TPI) {
    while (t < t1) {
      const long long item = t / TPI;
      q0 = static_cast<int>(t - item * TPI);
      q1 = t1 - t < TPI - q0 ? q0 + static_cast<int>(t1 - t) : TPI;
      t += q1 - q0;
      r = static_cast<int>(item / a.Hkv);
      g = static_cast<int>(item - static_cast<long long>(r) * a.Hkv);
      s = seq_info(a, r);
      if (s.ok) return true;
    }
    return false;
  }
};

template <int D, int CL>
struct FusedSmem {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t kKChunk = kFKRows * kRowBytes;     // one 64-channel chunk of K
  static constexpr uint32_t kKBytes = NCH * kKChunk;
  static constexpr uint32_t kQChunk = kFQRows * kRowBytes;
  static constexpr uint32_t kPAtom = 64 * kFQRows * 2;         // 64 keys x 128 queries, fp16
  static constexpr uint32_t kPBytes = 2 * kPAtom;
  static constexpr uint32_t kWBytes = 2 * 16 * kRowBytes;      // [k chunk][16 n rows][128 B]
  static constexpr int kQSlots = fq_slots(CL);
  static constexpr uint32_t kXBytes = kFXStages * CL * kFQRows * 4;   // [stage][rank][row]
  static constexpr uint32_t k_off = 0;
  static constexpr uint32_t q_off = k_off + kKBytes;            // [slot] one chunk each
  static constexpr uint32_t p_off = q_off + kQSlots * kQChunk;
  static constexpr uint32_t w_off = p_off + kFPBufs * kPBytes;
  static constexpr uint32_t x_off = w_off + kFPBufs * kWBytes;
  static constexpr uint32_t bar_off = x_off + kXBytes;
  static constexpr uint32_t kBars = 2 + 2 * kQSlots + 2 * kFTeams + 3 * kFPBufs + 2 * 2 + kFXStages;
  static constexpr uint32_t end = bar_off + kBars * 8 + 16;
  static constexpr size_t bytes = 1024 + end;
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Byte offset of (n, k) in a K-major 128-byte-swizzled 16-row B operand [k chunk][n][128 B].
__device__ __forceinline__ uint32_t w_offset(int n, int k) {
  return static_cast<uint32_t>((k >> 6) * 2048 + n * 128 + ((((k & 63) >> 3) ^ (n & 7)) << 4) +
                               (k & 7) * 2);
}

template <int D, int CL, bool PARTIAL, bool AGGMAX>
__global__ void __launch_bounds__(kFThreads, 1)
score_fused_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  // with a helper: it may start now, on the SMs this grid leaves idle
  if (a.done_count != nullptr) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using L = FusedSmem<D, CL>;
  constexpr int kFQSlots = L::kQSlots;
  constexpr int NCH = L::NCH;
  constexpr uint32_t kPageBytes = 16 * kRowBytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* k_buf = smem + L::k_off;
  uint8_t* q_buf = smem + L::q_off;
  uint8_t* p_buf = smem + L::p_off;
  uint8_t* w_buf = smem + L::w_off;
  float* x_buf = reinterpret_cast<float*>(smem + L::x_off);       // [stage][src rank][row]: lse
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bar_off);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + 1;
  uint64_t* q_full = bars + 2;                     // [kFQSlots]
  uint64_t* q_empty = q_full + kFQSlots;
  uint64_t* s_full = q_empty + kFQSlots;           // [kFTeams]
  uint64_t* s_empty = s_full + kFTeams;
  uint64_t* p_full = s_empty + kFTeams;            // [kFPBufs]
  uint64_t* w_full = p_full + kFPBufs;
  uint64_t* p_empty = w_full + kFPBufs;
  uint64_t* d_full = p_empty + kFPBufs;            // [2]
  uint64_t* d_empty = d_full + 2;
  uint64_t* x_full = d_empty + 2;                  // [kFXStages]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  // query tiles per head: CL = ceil(W / 128) (a cluster of 16 serves W = 2048 only); this
  // CTA's window keys: 128, fewer in the last CTA when W is not a multiple of 128 (PARTIAL,
  // an instantiation of its own so that the other windows' code stays as it is)
  constexpr int QT = CL;
  const int TPI = a.G * QT;
  const int kcount = PARTIAL ? min(kFKeys, a.W - static_cast<int>(rank) * kFKeys) : kFKeys;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    for (int i = 0; i < kFQSlots; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kFPBufs; ++i) {
      mbar_init(&p_full[i], kFTeamThreads);         // one team per tile
      mbar_init(&w_full[i], kFTeamThreads);
      mbar_init(&p_empty[i], AGGMAX ? kFTeamThreads : 1);   // the product, or the team
    }
    for (int i = 0; i < kFTeams; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kFTeamThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kFTeamThreads);       // the team that reads the segment's sums
    }
    for (int i = 0; i < kFXStages; ++i) mbar_init(&x_full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp >= 4) {
    // the weight operands' unused rows (n = 3 .. 15) stay zero
    constexpr int kZ = 16 - 3;
    const int t = threadIdx.x - 128;
    for (int i = t; i < kFPBufs * 2 * kZ * 8; i += kFEpiThreads) {
      const int buf = i / (16 * kZ), rem = i % (16 * kZ), kc = rem / (8 * kZ);
      const int n = 3 + (rem % (8 * kZ)) / 8, c = rem % 8;
      *reinterpret_cast<uint4*>(w_buf + buf * L::kWBytes + kc * 2048 + n * 128 + c * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();     // every CTA's barriers exist before any peer signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // rows of invalid sequences: zero scores, reported (this cluster's share of them)
    for (int r = cid * CL + static_cast<int>(rank); r < a.R; r += ncl * CL) {
      if (seq_info(a, r).ok) continue;
      for (int i = lane; i < a.Hkv * a.W; i += 32) a.scores[static_cast<size_t>(r) * a.Hkv * a.W + i] = 0.f;
      if (lane == 0) report(a.status, KARA_ERR_INVALID_ARG);
    }
    // ---- TMA producer: the item's key pages, then its query tiles; the next item's page
    // ids are fetched while this item's tiles stream ----
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
    }
    SegCursor cur;
    cur.init(a, cid, ncl, TPI);
    int C = 0;   // query chunks issued
    bool have = cur.next(a, TPI);
    auto page_ids = [&](const SeqInfo& s, int& npg) {
      const int key0 = s.start + static_cast<int>(rank) * kFKeys;
      npg = kcount <= 0 ? 0 : (key0 + kcount - 1) / 16 - key0 / 16 + 1;   // 8 or 9 when full
      return lane < npg ? page_block(a, s.b, key0 / 16 + lane) : 0;
    };
    int npg = 0;
    int my_blk = have ? page_ids(cur.s, npg) : 0;
    for (int I = 0; have; ++I) {
      if (__shfl_sync(0xffffffffu, *abort_flag != 0 ? 1 : 0, 0)) break;
      const int r = cur.r, gi = cur.g, q0 = cur.q0, q1 = cur.q1;
      const SeqInfo si = cur.s;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(k_empty, (I & 1) ^ 1, abort_flag, a.status) ? 1 : 0;
        if (ok) mbar_expect_tx(k_full, npg * NCH * kPageBytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int p = 0; p < npg; ++p) {
        const int blk = __shfl_sync(0xffffffffu, my_blk, p);
        if (lane == 0)
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_4d(k_buf + ch * L::kKChunk + p * kPageBytes, &tm_k, k_full, ch * 64, gi, 0, blk);
      }
      // the next segment's page ids (their loads overlap this segment's query tiles)
      have = cur.next(a, TPI);
      if (have) my_blk = page_ids(cur.s, npg);
      bool stop = false;
      if (lane == 0) {
        for (int tq = q0; tq < q1 && !stop; ++tq) {
          const int h = gi * a.G + tq / QT, qt = tq % QT;
          // L2 prefetch of the query tile fq_ahead(CL) tiles on (the CTAs of the cluster take
          // turns; the others' loads of it then hit L2)
          const int tp = tq + fq_ahead(CL);
          if (fq_ahead(CL) > 0 && tp < q1 && tq % CL == static_cast<int>(rank)) {
            const int hp = gi * a.G + tp / QT, qp = tp % QT;
            for (int ch = 0; ch < NCH; ++ch)
              tma_prefetch_l2_4d(&tm_q, ch * 64, hp, q_tile_row(a, si, qp * kFQRows),
                                 q_tile_batch(a, si, r));
          }
          for (int ch = 0; ch < NCH; ++ch) {   // chunk C of the ring: slot C mod 3
            const int slot = C % kFQSlots;
            if (!mbar_wait(&q_empty[slot], ((C / kFQSlots) & 1) ^ 1, abort_flag, a.status)) {
              stop = true;
              break;
            }
            mbar_expect_tx(&q_full[slot], L::kQChunk);
            tma_load_4d(q_buf + slot * L::kQChunk, &tm_q, &q_full[slot], ch * 64, h,
                        q_tile_row(a, si, qt * kFQRows), q_tile_batch(a, si, r));
            ++C;
          }
        }
      }
      C = __shfl_sync(0xffffffffu, C, 0);
      if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) break;
    }
  } else if (warp == 1) {
    // ---- UMMA issuer for S: runs ahead of the epilogue by one tile ----
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kFKeys);
      SegCursor cur;
      cur.init(a, cid, ncl, TPI);
      int T = 0, I = 0, C = 0;   // tiles, segments, query chunks
      bool ok = true;
      for (; ok && !*abort_flag && cur.next(a, TPI); ++I) {
        if (!mbar_wait(k_full, I & 1, abort_flag, a.status)) break;
        // the S product starts at the CTA's first key, row `off` of the loaded pages
        const int koff = (cur.s.start + static_cast<int>(rank) * kFKeys) % 16;
        const uint32_t k_addr = smem_u32(k_buf) + koff * kRowBytes;
        for (int tq = cur.q0; tq < cur.q1 && ok; ++tq, ++T) {
          const int st = T % kFTeams;
          const uint32_t ph = (T / kFTeams) & 1;
          if (!mbar_wait(&s_empty[st], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
          const uint32_t d_tmem = tmem_base + st * kFSCols;
          for (int ch = 0; ch < NCH; ++ch, ++C) {
            const int slot = C % kFQSlots;
            if (!mbar_wait(&q_full[slot], (C / kFQSlots) & 1, abort_flag, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(q_buf + slot * L::kQChunk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(q_addr + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(k_addr + ch * L::kKChunk + kk * 32);
              umma_bf16(d_tmem, ad, bd, idesc_s, (ch > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&q_empty[slot]);
          }
          if (!ok) break;
          umma_commit(&s_full[st]);
          if (tq == cur.q1 - 1) umma_commit(k_empty);
        }
      }
    }
  } else if (warp == 2 && !AGGMAX) {
    // ---- UMMA issuer for the column sums: D += P'^T W, tile by tile ----
    if (lane == 0) {
      const uint32_t idesc_c = idesc_f16_f32(128, 16, true);
      SegCursor cur;
      cur.init(a, cid, ncl, TPI);
      int Tc = 0, Ic = 0;
      for (; !*abort_flag && cur.next(a, TPI); ++Ic) {
        bool ok = true;
        for (int qt = cur.q0; qt < cur.q1; ++qt, ++Tc) {
          const int st = Tc % kFPBufs;
          const uint32_t ph = (Tc / kFPBufs) & 1;
          if (!mbar_wait(&p_full[st], ph, abort_flag, a.status) ||
              !mbar_wait(&w_full[st], ph, abort_flag, a.status) ||
              (qt == cur.q0 &&
               !mbar_wait(&d_empty[Ic & 1], ((Ic >> 1) & 1) ^ 1, abort_flag, a.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t p_addr = smem_u32(p_buf + st * L::kPBytes);
          const uint32_t w_addr = smem_u32(w_buf + st * L::kWBytes);
          const uint32_t d_tmem = tmem_base + kFDCol + (Ic & 1) * 16;
#pragma unroll
          for (int ks = 0; ks < kFQRows / 16; ++ks) {
            const uint64_t ad = sw128_mnmajor_desc(p_addr + ks * 2048, L::kPAtom, 1024);
            const uint64_t bd = sw128_kmajor_desc(w_addr + (ks >> 2) * 2048 + (ks & 3) * 32);
            umma_bf16(d_tmem, ad, bd, idesc_c, (ks > 0 || qt > cur.q0) ? 1u : 0u);
          }
          umma_commit(&p_empty[st]);
          if (qt == cur.q1 - 1) umma_commit(&d_full[Ic & 1]);
        }
        if (!ok) break;
      }
    }
  } else if (warp >= 4) {
    // ---- epilogue: three teams of 4 warps take the tiles in turn (team = tile mod 3), so
    // that a team's exchange wait and weights overlap the other teams' exponentials. In a
    // team, warp `quad` owns TMEM lane quadrant `quad`: each thread one query row and all
    // 128 keys of this CTA. ----
    const int e = warp - 4;
    const int team = e >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const float2 cs2 = make_float2(a.cs, a.cs);
    const uint32_t x_full_u32 = smem_u32(x_full);
    const uint32_t x_buf_u32 = smem_u32(x_buf);
    // warp-uniform bounded waits (a wait that gives up marks the whole warp aborted)
    bool aborted = false;
    auto wait_cta = [&](uint64_t* bar, uint32_t parity) {
      const bool ok = aborted ? false : mbar_wait(bar, parity, abort_flag, a.status);
      aborted = __any_sync(0xffffffffu, !ok) != 0;
    };
    auto wait_cluster = [&](uint64_t* bar, uint32_t parity) {
      const bool ok = aborted ? false : mbar_wait_cluster(bar, parity, abort_flag, a.status);
      aborted = __any_sync(0xffffffffu, !ok) != 0;
    };
    SegCursor cur;
    cur.init(a, cid, ncl, TPI);
    int I = 0, tp = team;                 // segment index and tile within the segment (no
    bool have = cur.next(a, TPI);         // divisions per tile: they would queue behind the
    while (have && tp >= cur.q1 - cur.q0) {   // exponentials)
      tp -= cur.q1 - cur.q0;
      ++I;
      have = cur.next(a, TPI);
    }
    // this team's buffers: S, P' and weights `team`, used every third tile (phase = T div 3);
    // exchange slot T mod 6 (xs) and its phase T div 6 (xq)
    const int st = team;
    uint8_t* const prow = p_buf + st * L::kPBytes + (row >> 3) * 1024 + (row & 7) * 128;
    uint32_t sq = 0;
    int xs = team, xq = 0;
    float kmax0 = 0.f, kmax1 = 0.f;   // the max aggregation: this thread's two keys
    for (int T = team; have; T += kFTeams, ++sq) {
      const uint32_t ph = sq & 1;
      const uint32_t scol = lane_base + st * kFSCols;
      // (1) row max over this CTA's 128 keys (first pass over TMEM)
      wait_cta(&s_full[st], ph);
      float mx = 0.f, l = 0.f;
      if (!aborted) {
        tc_fence_after();
        if (PARTIAL && kcount < kFKeys) {
          // keys past the window (the last CTA of a window that is not a multiple of 128):
          // their S columns become -inf, so that they set no row max and give P' = 0. Single
          // columns up to a multiple of 16, then 16 at a time (past column 128 + offset lie
          // columns the passes do not read).
          uint32_t c = scol + kcount;
          const uint32_t c_end = scol + kFKeys;
#pragma unroll 1
          for (; (c & 15u) != 0 && c < c_end; ++c) tmem_st1(c, -INFINITY);
#pragma unroll 1
          for (; c < c_end; c += 16) tmem_st16_fill(c, -INFINITY);
          tmem_wait_st();
        }
        float v[32];
        float mm = -INFINITY;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          tmem_ld16(scol + 32 * h, v);
          tmem_ld16(scol + 32 * h + 16, v + 16);
          tmem_wait_ld();
          reg_fence<32>(v);
          float mq[11];
#pragma unroll
          for (int q = 0; q < 10; ++q) mq[q] = fmax3(v[3 * q], v[3 * q + 1], v[3 * q + 2]);
          mq[10] = fmaxf(v[30], v[31]);
          const float m0 = fmax3(mq[0], mq[1], mq[2]), m1 = fmax3(mq[3], mq[4], mq[5]);
          const float m2 = fmax3(mq[6], mq[7], mq[8]), m3 = fmax3(mq[9], mq[10], mm);
          mm = fmaxf(fmax3(m0, m1, m2), m3);
        }
        mx = mm == -INFINITY ? 0.f : mm * a.cs;   // a CTA without keys: P' = 0, lse = -inf
        wait_cta(&p_empty[st], ph ^ 1);
      }
      // (2) P' = 2^(s c - m + 15) as fp16 in shared memory (second pass), and the row sum;
      // keys [32 h, 32 h + 32) go to atom h / 2, granules 4 (h mod 2) .. + 3
      if (!aborted) {
        const float2 nb2 = make_float2(15.f - mx, 15.f - mx);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float v[32];
          tmem_ld16(scol + 32 * h, v);
          tmem_ld16(scol + 32 * h + 16, v + 16);
          tmem_wait_ld();
          reg_fence<32>(v);
          if (h == 3) {
            tc_fence_before();
            mbar_arrive(&s_empty[st]);
          }
          uint8_t* patom = prow + (h >> 1) * L::kPAtom;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 8; i += 4) {
              const int j = 8 * c + i;
              const float2 x0 = ffma2(make_float2(v[j], v[j + 1]), cs2, nb2);
              const float2 x1 = ffma2(make_float2(v[j + 2], v[j + 3]), cs2, nb2);
              const float2 e0 = make_float2(ex2(x0.x), ex2(x0.y));
              const float2 e1 = make_float2(ex2(x1.x), ex2(x1.y));
              acc0 = fadd2(acc0, e0);
              acc1 = fadd2(acc1, e1);
              pk[i / 2] = pack_f16x2(e0.x, e0.y);
              pk[i / 2 + 1] = pack_f16x2(e1.x, e1.y);
            }
            const int cc = 4 * (h & 1) + c;
            *reinterpret_cast<uint4*>(patom + ((cc ^ (row & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        l = (acc0.x + acc0.y) + (acc1.x + acc1.y);
        fence_proxy_async();
        mbar_arrive(&p_full[st]);
      }
      // (3) the CTA's partial log-sum-exp of the row to every CTA of the cluster
      if ((e & 3) == 0 && lane == 0) mbar_expect_tx(&x_full[xs], CL * kFQRows * 4);
      if (!aborted) {
        const float lse = mx + lg2(l);
        const uint32_t slot = x_buf_u32 + ((xs * CL + rank) * kFQRows + row) * 4;
        const uint32_t xb = x_full_u32 + xs * 8;
#pragma unroll
        for (int c = 0; c < CL; ++c) st_async_f32(map_to_rank(slot, c), lse, map_to_rank(xb, c));
      }
      // (4) once every CTA's partials are in: the row weight w = 2^(m - M + 15) / L as three
      // fp16 columns of the B operand
      wait_cluster(&x_full[xs], xq & 1);
      if (!aborted) {
        const float* xr = x_buf + xs * CL * kFQRows + row;
        float xv[CL];
#pragma unroll
        for (int c = 0; c < CL; ++c) xv[c] = xr[c * kFQRows];
        float M = xv[0];
#pragma unroll
        for (int c = 1; c < CL; ++c) M = fmaxf(M, xv[c]);
        float Lsum = 0.f;
#pragma unroll
        for (int c = 0; c < CL; ++c) Lsum += ex2(xv[c] - M);
        float inv;   // 1 / L to about 2^-23 (rcp.approx), well inside the score tolerance
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(Lsum));
        float w = ex2(mx - M + 15.f) * inv;
        // query rows past the window (the last tile of a window that is not a multiple of
        // 128): weight 0
        if (PARTIAL && ((cur.q0 + tp) % QT) * kFQRows + row >= a.W) w = 0.f;
        if (AGGMAX) {
          // the row's softmax factor, P' w / 2^15, for the column maxima below
          reinterpret_cast<float*>(w_buf + st * L::kWBytes)[row] = w * (1.f / 32768.f);
        } else {
          const __half w1 = __float2half_rn(w);
          const float r1 = w - __half2float(w1);
          const __half w2 = __float2half_rn(r1);
          const float r2 = r1 - __half2float(w2);
          const __half w3 = __float2half_rn(r2 * 16777216.f);
          uint8_t* wb = w_buf + st * L::kWBytes;
          *reinterpret_cast<__half*>(wb + w_offset(0, row)) = w1;
          *reinterpret_cast<__half*>(wb + w_offset(1, row)) = w2;
          *reinterpret_cast<__half*>(wb + w_offset(2, row)) = w3;
          fence_proxy_async();
          mbar_arrive(&w_full[st]);
        }
      }
      if (AGGMAX) {
        // (4') the max aggregation: per key, the largest softmax value over the tile's rows,
        // from P' in shared memory times the row factors (thread: keys 2p, 2p + 1 of this
        // CTA, rows 64 h .. 64 h + 63); kept in registers over the team's tiles of the
        // segment, then merged into the output with an atomic max (non-negative floats order
        // as their bits)
        named_barrier(1 + team, kFTeamThreads);     // the team's P' rows and factors are in
        const int kp = row & 63, rh = row >> 6;
        if (!aborted) {
          const float* wr = reinterpret_cast<const float*>(w_buf + st * L::kWBytes);
          const uint8_t* pb = p_buf + st * L::kPBytes + (kp >> 5) * L::kPAtom + 4 * (kp & 3);
          const int gq = (kp & 31) >> 2;               // the keys' 16-byte granule in a row
          float m0 = 0.f, m1 = 0.f;
          const float2 zero2 = make_float2(0.f, 0.f);
#pragma unroll 4
          for (int i = 64 * rh; i < 64 * rh + 64; i += 2) {   // two rows at a time
            const uint32_t pa = *reinterpret_cast<const uint32_t*>(
                pb + (i >> 3) * 1024 + (i & 7) * 128 + ((gq ^ (i & 7)) << 4));
            const uint32_t pc = *reinterpret_cast<const uint32_t*>(
                pb + (i >> 3) * 1024 + ((i + 1) & 7) * 128 + ((gq ^ ((i + 1) & 7)) << 4));
            const float2 wi = *reinterpret_cast<const float2*>(wr + i);
            const float2 fa = ffma2(__half22float2(*reinterpret_cast<const __half2*>(&pa)),
                                    make_float2(wi.x, wi.x), zero2);
            const float2 fc = ffma2(__half22float2(*reinterpret_cast<const __half2*>(&pc)),
                                    make_float2(wi.y, wi.y), zero2);
            m0 = fmax3(m0, fa.x, fc.x);
            m1 = fmax3(m1, fa.y, fc.y);
          }
          kmax0 = fmaxf(kmax0, m0);
          kmax1 = fmaxf(kmax1, m1);
        }
        mbar_arrive(&p_empty[st]);                  // this thread is done with P'
        if (tp + kFTeams >= cur.q1 - cur.q0) {      // the team's last tile of the segment
          if (!aborted) {
            float* dst;
            if (cur.q0 == 0 && cur.q1 == TPI) {
              dst = a.scores + (static_cast<size_t>(cur.r) * a.Hkv + cur.g) * a.W;
            } else {
              const int side = cur.q0 == 0 ? 0 : 1;
              const int split = side == 0 ? cid + 1 : cid;
              dst = a.part + (static_cast<size_t>(split - 1) * 2 + side) * a.W;
            }
            const int k0 = static_cast<int>(rank) * kFKeys + 2 * kp;
            if (!PARTIAL || 2 * kp < kcount)
              atomicMax(reinterpret_cast<unsigned int*>(dst + k0), __float_as_uint(kmax0));
            if (!PARTIAL || 2 * kp + 1 < kcount)
              atomicMax(reinterpret_cast<unsigned int*>(dst + k0 + 1), __float_as_uint(kmax1));
          }
          kmax0 = 0.f;
          kmax1 = 0.f;
        }
      }
      // (5) the segment's last tile: the per-key sums over its heads, read by this team
      if (!AGGMAX && tp == cur.q1 - cur.q0 - 1) {
        wait_cta(&d_full[I & 1], (I >> 1) & 1);
        if (!aborted) {
          tc_fence_after();
          // TMEM lane `row` of D holds key `row` of this CTA
          float d[4];
          tmem_ld4(lane_base + kFDCol + (I & 1) * 16, d);
          tmem_wait_ld();
          reg_fence<4>(d);
          const float val =
              (d[0] + d[1] + d[2] * (1.f / 16777216.f)) * (1.f / 32768.f) * a.out_scale;
          float* dst;
          if (cur.q0 == 0 && cur.q1 == TPI) {
            dst = a.scores + (static_cast<size_t>(cur.r) * a.Hkv + cur.g) * a.W;
          } else {   // the head part ends this cluster's range (split cid + 1), the tail
                     // part starts it (split cid)
            const int side = cur.q0 == 0 ? 0 : 1;
            const int split = side == 0 ? cid + 1 : cid;
            dst = a.part + (static_cast<size_t>(split - 1) * 2 + side) * a.W;
          }
          if (!PARTIAL || static_cast<int>(rank) * kFKeys + row < a.W) dst[rank * kFKeys + row] = val;
          tc_fence_before();
          mbar_arrive(&d_empty[I & 1]);
        }
      }
      xs += kFTeams;
      if (xs >= kFXStages) { xs -= kFXStages; ++xq; }
      tp += kFTeams;
      while (have && tp >= cur.q1 - cur.q0) {
        tp -= cur.q1 - cur.q0;
        ++I;
        have = cur.next(a, TPI);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  cluster_sync_all();     // no CTA leaves while a peer may still write into its shared memory
  if (a.done_count != nullptr && threadIdx.x == 0) {
    __threadfence();      // this CTA's writes (ordered by the barrier above) before the count
    atomicAdd(a.done_count, 1);
  }
}

// Items split between two clusters of the fused kernel: scores = head part + tail part (in
// that order, so the result does not depend on which part finished first). One CTA per
// range boundary k = 1 .. ncl - 1; boundaries on an item boundary have nothing to add.
__global__ void __launch_bounds__(256)
score_split_sum_kernel(const ScoreArgs a, int ncl, int TPI) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the fused kernel's writes are visible
  const int k = blockIdx.x + 1;
  const long long n = a.items * TPI;
  const long long t = k * n / ncl;
  const long long item = t / TPI;
  if (t == item * TPI) return;
  const int r = static_cast<int>(item / a.Hkv);
  const int g = static_cast<int>(item - static_cast<long long>(r) * a.Hkv);
  if (!seq_info(a, r).ok) return;
  const float* head = a.part + static_cast<size_t>(k - 1) * 2 * a.W;
  const float* tail = head + a.W;
  float* dst = a.scores + (static_cast<size_t>(r) * a.Hkv + g) * a.W;
  for (int j = threadIdx.x; j < a.W; j += blockDim.x)
    dst[j] = a.max_agg ? fmaxf(head[j], tail[j]) : head[j] + tail[j];
}

template <int D>
constexpr size_t rowstats_smem() {
  return 1024 + 2 * (D / 64) * kKRows1 * kRowBytes + kQStages1 * (D / 64) * kQRows1 * kRowBytes +
         3 * kQRows1 * sizeof(float2) + 256;
}
template <int D>
constexpr size_t colsum_smem() {
  return 1024 + 2 * (D / 64) * kKRows2 * kRowBytes + kQStages2 * (D / 64) * kQRows2 * kRowBytes +
         (2 * kQRows2 + 3 * kKRows2) * sizeof(float) + 256;
}

// Appends the kernel's resource attributes to the last-error text (after a refused launch).
void describe_kernel(const char* name, const void* fn, int threads, size_t dyn_smem) {
  cudaFuncAttributes at;
  char buf[400];
  if (cudaFuncGetAttributes(&at, fn) == cudaSuccess) {
    std::snprintf(buf, sizeof(buf),
                  "launch refused: %d threads, %zu B dynamic smem; kernel uses %d regs, max %d "
                  "threads/block, %zu B static smem, max dynamic smem %d B",
                  threads, dyn_smem, at.numRegs, at.maxThreadsPerBlock, at.sharedSizeBytes,
                  at.maxDynamicSharedSizeBytes);
    set_last_error(name, buf);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 4-D bf16 tensor map, innermost dimension first, 128-byte swizzle, box {64, 1, rows, 1}.
bool make_map(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
              uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gdim[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gstride[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t box[4] = {64, 1, box_rows, 1};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim, gstride,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

// SMs of device slot `dev` (queried once per device).
int sm_count(int dev) {
  static std::atomic<int> count[kMaxDevices];
  int n = count[dev].load();
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    count[dev].store(n);
  }
  return n;
}

// The helper: items [item0, item0 + h) on F CTAs (one per idle SM), as the fused kernel's
// programmatic dependent; CTA 0 waits for `target` fused CTAs at its end.
template <int D>
kara_status launch_helper(ScoreArgs a, const ScoreLaunch& L, const CUtensorMap& tq1,
                          const CUtensorMap& tq2, const CUtensorMap& tk, long long item0,
                          long long h, int F, int target, cudaStream_t stream) {
  static std::atomic<int> attr_done[kMaxDevices];   // per device: the smem limit is set
  const int dev = device_slot();
  constexpr size_t smem = rowstats_smem<D>() > colsum_smem<D>() ? rowstats_smem<D>()
                                                               : colsum_smem<D>();
  if (!attr_done[dev].load()) {
    cudaFuncSetAttribute(score_item_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    attr_done[dev].store(1);
  }
  a.lse = L.lse;
  a.done_target = target;
  launch_pdl(score_item_kernel<D>, dim3(F), dim3(kThreads), smem, stream, tq1, tq2, tk, a,
             item0, h);
  if (check_launch("score_item_kernel") != KARA_OK) {
    describe_kernel("score_item_kernel", reinterpret_cast<const void*>(score_item_kernel<D>),
                    kThreads, smem);
    return KARA_ERR_CUDA;
  }
  return KARA_OK;
}

template <int D>
kara_status launch_score(const ScoreLaunch& L, cudaStream_t stream) {
  // queries: q_win [R, W, Hq, d], or the window-query ring [batch, 2W, Hq, d]
  const uint64_t qrows = static_cast<uint64_t>(L.ring ? 2 * L.W : L.W);
  const uint64_t qdims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(L.Hq), qrows,
                             static_cast<uint64_t>(L.ring ? L.batch : L.R)};
  const uint64_t qstr[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(L.Hq) * D * 2,
                            qrows * L.Hq * D * 2};
  const uint64_t kdims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(L.Hkv), 16,
                             static_cast<uint64_t>(L.num_blocks)};
  const uint64_t kstr[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(L.Hkv) * D * 2,
                            static_cast<uint64_t>(16) * L.Hkv * D * 2};
  CUtensorMap tq1, tq2, tk;
  if (!make_map(&tq1, L.q_win, qdims, qstr, kQRows1) ||
      !make_map(&tq2, L.q_win, qdims, qstr, kQRows2) || !make_map(&tk, L.k_cache, kdims, kstr, 16)) {
    set_last_error("kara_score", "cuTensorMapEncodeTiled failed");
    return KARA_ERR_CUDA;
  }

  ScoreArgs a;
  a.block_table = L.block_table;
  a.ctx_len = L.ctx_len;
  a.seq_ids = L.seq_ids;
  a.lse = L.lse;
  a.lse_merged = L.lse + static_cast<size_t>(L.R) * L.Hq * score_chunks(L.W) * score_lse_stride(L.W);
  a.scores = L.scores;
  a.status = L.status;
  a.R = L.R;
  a.W = L.W;
  a.Wp = score_lse_stride(L.W);
  a.CM = score_chunks(L.W);
  a.Hq = L.Hq;
  a.Hkv = L.Hkv;
  a.G = L.Hq / L.Hkv;
  a.batch = L.batch;
  a.max_blocks = L.max_blocks;
  a.num_blocks = L.num_blocks;
  a.cs = L.scale * 1.4426950408889634f;
  a.ring = L.ring;
  a.part = nullptr;
  a.streamk = 0;
  a.out_scale = L.agg == KARA_AGG_MEAN ? 1.f / (static_cast<float>(a.G) * L.W) : 1.f;
  a.max_agg = 0;
  a.row0 = 0;
  a.g0 = 0;
  a.HkvN = L.Hkv;
  a.items = static_cast<long long>(L.R) * L.Hkv;
  a.done_count = nullptr;
  a.done_target = 0;
  const bool agg_max = L.agg == KARA_AGG_MAX;
  const int dev = device_slot();
  if (dev < 0) {
    set_last_error("kara_score", "no usable current CUDA device");
    return KARA_ERR_CUDA;
  }


  // Windows of up to 1024 keys, and of 2048: the fused single-exponential kernel on clusters
  // of ceil(W / 128) CTAs (the max aggregation: head_dim 128 and up to 1024 keys). A cluster
  // of 16 is non-portable: where the device cannot hold one, W = 2048 takes the two-pass path
  // too, as do the other windows.
  // per device, cluster size, partial last CTA and aggregation: resident clusters, queried
  // once (-1: none fits)
  static std::atomic<int> max_clusters[kMaxDevices][kFMaxCluster + 1][2][2];
  const int CL = (L.W + kFKeys - 1) / kFKeys;            // query tiles per head too
  const int PT = L.W % kFKeys != 0 ? 1 : 0;             // the last CTA owns fewer keys
  const int AG = agg_max ? 1 : 0;
  const bool fused_window = agg_max ? (D == 128 && L.W >= 1 && L.W <= 8 * kFKeys)
                                    : (L.W >= 1 && L.W <= 8 * kFKeys) || L.W == kFMaxCluster * kFKeys;
  if (fused_window && max_clusters[dev][CL][PT][AG].load() >= 0) {
    using KernT = void (*)(CUtensorMap, CUtensorMap, ScoreArgs);
    KernT kern = nullptr;
    size_t smem = 0;
    switch (CL) {
#define KARA_FUSED_CASE(c)                                                                  \
      case c:                                                                               \
        if constexpr (D == 128) {                                                           \
          if (AG) {                                                                         \
            kern = PT ? score_fused_kernel<D, c, true, true> : score_fused_kernel<D, c, false, true>; \
            smem = FusedSmem<D, c>::bytes;                                                  \
            break;                                                                          \
          }                                                                                 \
        }                                                                                   \
        kern = PT ? score_fused_kernel<D, c, true, false> : score_fused_kernel<D, c, false, false>; \
        smem = FusedSmem<D, c>::bytes;                                                      \
        break;
      KARA_FUSED_CASE(1) KARA_FUSED_CASE(2) KARA_FUSED_CASE(3) KARA_FUSED_CASE(4)
      KARA_FUSED_CASE(5) KARA_FUSED_CASE(6) KARA_FUSED_CASE(7) KARA_FUSED_CASE(8)
#undef KARA_FUSED_CASE
      default:
        kern = score_fused_kernel<D, 16, false, false>;
        smem = FusedSmem<D, 16>::bytes;
        break;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // kernel waits at entry
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (max_clusters[dev][CL][PT][AG].load() == 0) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
      if (CL > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      cfg.gridDim = dim3(CL * (sm_count(dev) / CL));
      cfg.numAttrs = 1;                    // the query sees the cluster shape only
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      cfg.numAttrs = 2;
      if (qe != cudaSuccess || n <= 0) {
        if (CL <= 8) {
          check_launch("score_fused_kernel occupancy");
          return KARA_ERR_CUDA;
        }
        cudaGetLastError();                // no cluster of 16 fits: the two-pass path below
        n = -1;
      }
      max_clusters[dev][CL][PT][AG].store(n);
    }
    if (max_clusters[dev][CL][PT][AG].load() > 0) {
      const int maxc = max_clusters[dev][CL][PT][AG].load();
      const long long all_items = static_cast<long long>(L.R) * L.Hkv;
      const size_t ws_bytes = score_workspace_bytes(L.R, L.W, L.Hq);
      // Helper items: when the clusters fill the GPU and leave at least kHelperMinSms SMs
      // idle, score_item_kernel takes the last m * F items there (F = the idle SMs, m items
      // each), m from the per-SM cost of an item on the two-pass path against the fused one
      // (kHelperCost: 2.5 on clusters of up to 8, 2.0 on clusters of 16, measured), so that
      // both kernels end together. Sum and mean, head_dim 128. Workspace: [F one-row two-pass
      // regions][split parts][done counter].
      const int F = sm_count(dev) - maxc * CL;
      long long h = 0;
      if (!AG && D == 128 && F >= kHelperMinSms && all_items >= maxc) {
        const double cost = CL > 8 ? kHelperCost16 : kHelperCost;
        const long long m = static_cast<long long>(all_items / (cost * maxc * CL + F));
        h = m * F;
        const size_t need = static_cast<size_t>(F) * score_workspace_bytes(1, L.W, L.Hq) +
                            static_cast<size_t>(maxc - 1) * 2 * L.W * sizeof(float) + 16;
        if (all_items - h < maxc || need > ws_bytes) h = 0;
      }
      const long long items = all_items - h;
      a.items = items;
      const int ncl = static_cast<int>(
          std::max<long long>(1, std::min<long long>(maxc, items)));
      // Tile-granular ranges whenever the split slots fit in the workspace (they do whenever
      // ncl <= items, which the grid guarantees; checked all the same). The ranges are then at
      // least TPI tiles long, as the kernel assumes.
      const int TPI = a.G * CL;
      const long long ntiles = items * TPI;
      const size_t part_bytes = static_cast<size_t>(ncl - 1) * 2 * L.W * sizeof(float);
      const size_t helper_floats =
          h > 0 ? static_cast<size_t>(F) * score_workspace_bytes(1, L.W, L.Hq) / sizeof(float) : 0;
      a.part = L.lse + helper_floats;
      a.streamk = ncl > 1 && ntiles / ncl >= TPI &&
                  helper_floats * sizeof(float) + part_bytes <= ws_bytes;
      if (h > 0) {
        a.done_count = reinterpret_cast<int*>(a.part + static_cast<size_t>(ncl - 1) * 2 * L.W);
        if (cudaMemsetAsync(a.done_count, 0, sizeof(int), stream) != cudaSuccess) {
          check_launch("kara_score helper counter");
          return KARA_ERR_CUDA;
        }
      }
      a.max_agg = AG;
      if (AG) {
        // the max aggregation merges into zeroed outputs with atomic maxima (softmax >= 0)
        if (cudaMemsetAsync(L.scores, 0, static_cast<size_t>(L.R) * L.Hkv * L.W * sizeof(float),
                            stream) != cudaSuccess ||
            (a.streamk && cudaMemsetAsync(a.part, 0, part_bytes, stream) != cudaSuccess)) {
          check_launch("kara_score max zero fill");
          return KARA_ERR_CUDA;
        }
      }
      bool any_split = false;
      for (int k = 1; a.streamk && k < ncl && !any_split; ++k)
        any_split = (k * ntiles / ncl) % TPI != 0;
      cfg.gridDim = dim3(ncl * CL);
      count_launch(cudaLaunchKernelEx(&cfg, kern, tq1, tk, a));
      if (check_launch("score_fused_kernel") != KARA_OK) {
        describe_kernel("score_fused_kernel", reinterpret_cast<const void*>(kern), kFThreads, smem);
        return KARA_ERR_CUDA;
      }
      if (h > 0) {
        if constexpr (D == 128) {
          const kara_status hs = launch_helper<D>(a, L, tq1, tq2, tk, items, h, F, ncl * CL,
                                                  stream);
          if (hs != KARA_OK) return hs;
        }
      }
      if (any_split) {
        launch_pdl(score_split_sum_kernel, dim3(ncl - 1), dim3(256), 0, stream, a, ncl, TPI);
        if (check_launch("score_split_sum_kernel") != KARA_OK) return KARA_ERR_CUDA;
      }
      return KARA_OK;
    }
  }

  static std::atomic<int> attr_set[kMaxDevices];   // per device: the limits are set
  if (!attr_set[dev].load()) {
    cudaFuncSetAttribute(score_rowstats_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(rowstats_smem<D>()));
    cudaFuncSetAttribute(score_colsum_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(colsum_smem<D>()));
    cudaFuncSetAttribute(score_colsum_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(colsum_smem<D>()));
    attr_set[dev].store(1);
  }
  const int tiles1 = L.R * L.Hkv * score_chunks(L.W) * (L.Hq / L.Hkv);   // upper bound
  const int KT = ((L.W + 15 + 15) / 16 + 7) / 8;   // at most this many key tiles per (r, g)
  const int tiles2 = L.R * L.Hkv * KT;
  const int sms = sm_count(dev);
  launch_pdl(score_rowstats_kernel<D>, dim3(min(tiles1, sms)), dim3(kThreads), rowstats_smem<D>(),
             stream, tq1, tk, a);
  if (check_launch("score_rowstats_kernel") != KARA_OK) {
    describe_kernel("score_rowstats_kernel", reinterpret_cast<const void*>(score_rowstats_kernel<D>),
                    kThreads, rowstats_smem<D>());
    return KARA_ERR_CUDA;
  }
  {
    const size_t n = static_cast<size_t>(L.R) * L.Hq * score_lse_stride(L.W);
    const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, static_cast<size_t>(sms) * 8));
    launch_pdl(score_lse_merge_kernel, dim3(blocks), dim3(256), 0, stream, a);
    if (check_launch("score_lse_merge_kernel") != KARA_OK) return KARA_ERR_CUDA;
  }
  auto colsum = agg_max ? score_colsum_kernel<D, true> : score_colsum_kernel<D, false>;
  launch_pdl(colsum, dim3(min(tiles2, sms)), dim3(kThreads), colsum_smem<D>(), stream, tq2, tk,
             a);
  if (check_launch("score_colsum_kernel") != KARA_OK) {
    describe_kernel("score_colsum_kernel", reinterpret_cast<const void*>(colsum), kThreads,
                    colsum_smem<D>());
    return KARA_ERR_CUDA;
  }
  return KARA_OK;
}

}  // namespace

bool make_bf16_map_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                      const uint64_t strides[3], uint32_t box_rows) {
  return make_map(map, base, dims, strides, box_rows);
}

int score_lse_stride(int W) { return (W + 255) / 256 * 256; }

// 16-page key chunks a window of W slots can span (its pages: at most ceil((W + 15) / 16)).
int score_chunks(int W) { return ((W + 15 + 15) / 16 + 15) / 16; }

size_t score_workspace_bytes(int R, int W, int Hq) {
  return static_cast<size_t>(R) * Hq * (score_chunks(W) + 1) * score_lse_stride(W) * sizeof(float);
}

kara_status launch_score_kernels(const ScoreLaunch& L, cudaStream_t stream) {
  if (L.D == 128) return launch_score<128>(L, stream);
  if (L.D == 64) return launch_score<64>(L, stream);
  return KARA_ERR_UNSUPPORTED;
}

}  // namespace kara
