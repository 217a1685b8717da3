// Paged grouped-query decode attention over the (compressed) cache, split-KV.
//
// out[b][h] = sum_t softmax_t(q_bh . k_t * scale) v_t over the slots [0, ctx_len[b]) read
// through the block table ("Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache
// Compression", English abstract: the kept KV pairs serve subsequent decoding; the method is
// adapted to PagedAttention).
//
// HBM-bound: every K and V row of a KV head is loaded once for all G query heads of its group.
// Persistent kernel (CTAs of 4 warps, as many per SM as registers and shared memory allow);
// every warp is an independent stream over work units (sequence, KV head, 8-page split) and
// leaves one partial (m, l, unnormalised o) per unit and query head; a second kernel merges the
// partials of each (sequence, query head). Pages reach shared memory by TMA (one 16-row box of
// one KV head per 64 channels, 128-byte swizzle) through a per-warp ring of single pages that
// carries a unit's K pages, then its V pages, and keeps streaming across unit boundaries.
//
// The per-page products run on warp-level mma.sync (m16n8k16, bf16 in, fp32 accumulate) with
// the group's query heads as the 8-wide N side: with G = 7 heads a page costs 1792 FMAs per 256
// bytes of K and V, close to the point where CUDA-core issue rather than HBM binds, so the
// tensor cores here cut the instruction stream (about 40 per page instead of about 1400) rather
// than add arithmetic throughput.
#include <cuda.h>

#include <cstdint>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace kara {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = 4;
constexpr int kUnitPages = 8;      // pages per work unit (one partial per unit)

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* block_table;
  const int32_t* ctx_len;
  float* part_o;       // [B, Hq, S, D]: unnormalised o per split (16-byte aligned rows)
  float2* part_ml;     // [B, Hq, S]: (m, l) per split
  int32_t* status;
  int B, Hq, Hkv, max_blocks, num_blocks, S;
  float cs;            // scale * log2(e)
  // fused decode step (append): the new token of every sequence at slot n = ctx_len
  int append;
  const __nv_bfloat16* k_new;   // [B, Hkv, D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_dst;         // the caches the new token is written to (= k, v)
  __nv_bfloat16* v_dst;
  __nv_bfloat16* q_ring;        // [B, 2W, Hq, D] or null
  int ring_w;                   // W
};

template <int D>
__host__ __device__ constexpr int page_bytes() { return 16 * D * 2; }   // one page, one KV head
// Two ring shapes with the same bytes in flight per SM: DEEP = 3 CTAs per SM with 4-page rings
// per warp, else 4 CTAs per SM (128 registers a thread) with 3-page rings.
template <bool DEEP>
__host__ __device__ constexpr int dec_stages() { return DEEP ? 4 : 3; }   // ring depth, pages
template <bool DEEP>
__host__ __device__ constexpr int dec_min_blocks() { return DEEP ? 3 : 4; }

template <int D, bool DEEP>
constexpr size_t stream_smem_bytes() {
  // [warp][stage] one page (1024-aligned) + the warps' ring barriers
  return 1024 + static_cast<size_t>(kDecWarps) * dec_stages<DEEP>() * page_bytes<D>() +
         8 * dec_stages<DEEP>() * kDecWarps;
}

// Byte offset of 16-byte granule `gi` of row `r` in a 128-byte-swizzled 16-row box.
__device__ __forceinline__ uint32_t sw128(int r, int gi) {
  return static_cast<uint32_t>(r * 128 + ((gi ^ (r & 7)) << 4));
}

// Work units (b, split, g), g fastest: split s covers pages [8s, 8s+8) of sequence b. Warps
// with consecutive unit ids (the warps of one CTA) read the KV heads of the same blocks at about
// the same time, so each block's DRAM rows are fetched together.
struct Unit {
  int b, g, split, n, p0, np;   // np: pages of the unit
  bool ok;
};

struct UnitCursor {
  int b = 0, base = 0, per = -1, n = 0, npages = 0;
  __device__ __forceinline__ Unit seek(const DecodeArgs& a, int u) {
    Unit x;
    x.ok = false;
    while (true) {
      if (b >= a.B) return x;
      if (per < 0) {
        n = a.ctx_len[b];
        if (n > a.max_blocks * 16) {
          report(a.status, KARA_ERR_INVALID_ARG);
          n = a.max_blocks * 16;
        }
        if (n < 0) n = 0;
        npages = (n + 15) / 16;
        per = a.Hkv * ((npages + kUnitPages - 1) / kUnitPages);
      }
      if (u < base + per) break;
      base += per;
      ++b;
      per = -1;
    }
    const int local = u - base;
    x.b = b;
    x.g = local % a.Hkv;
    x.split = local / a.Hkv;
    x.n = n;
    x.p0 = x.split * kUnitPages;
    x.np = min(kUnitPages, npages - x.p0);
    x.ok = true;
    return x;
  }
};

// ldmatrix / movmatrix / mma.sync helpers (m16n8k16, bf16 inputs, fp32 accumulators).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Persistent, one independent stream per warp: the warp walks units u = warp_id, +num_warps,
// ...; its TMA ring (dec_stages single pages) streams, per unit, the unit's K pages and then its
// V pages, and keeps streaming across unit boundaries (the next unit's block ids and queries
// are fetched ahead). Every unit leaves one partial (m, l, o) per query head for the combine
// kernel.
//
// The G <= 8 query heads of the group are the N = 8 side of warp-level m16n8k16 products, so
// no fragment row is padding: per K page, S^T (16 slots x 8 heads) = K (16 x d) Q^T over d/16
// steps, with K fragments read from the swizzled page by ldmatrix and Q^T held in registers
// for the whole unit. The unit's scores stay in registers (4 per thread per page); one max per
// head over the unit fixes the exponent base, so the accumulators are never rescaled. P^T goes
// to bf16 and, transposed in registers by movmatrix, becomes the B operand of O^T (d x 8) +=
// V^T (d x 16) P^T (16 x 8), with V^T fragments read by ldmatrix.trans.
template <int D, int G, bool DEEP>
__global__ void __launch_bounds__(kDecThreads, dec_min_blocks<DEEP>())
decode_stream_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  static_assert(G <= 8, "at most 8 query heads per KV head");
  constexpr int kStages = dec_stages<DEEP>();
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  constexpr int NCH = D / 64;                 // 64-channel chunks per row
  constexpr int KS = D / 16;                  // k-steps of S^T, m-tiles of O^T
  constexpr uint32_t kPage = page_bytes<D>();
  constexpr uint32_t kChunkBytes = 16 * 128;  // one 64-channel chunk of a page
  const int warp = warp_id(), lane = lane_id();
  const int grp = lane >> 2, tig = lane & 3;  // fragment row / column pair
  const int mtx = lane >> 3, mrow = lane & 7; // ldmatrix: lane feeds row mrow of matrix mtx

  extern __shared__ __align__(1024) uint8_t dsm[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* my_ring = ring + static_cast<size_t>(warp) * kStages * kPage;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(ring + kDecWarps * kStages * kPage) +
                      warp * kStages;
  const uint32_t ring_u32 = smem_u32(my_ring);

  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&my_bars[st], 1);
    fence_barrier_init();
  }
  __syncthreads();
  // the combine kernel may be scheduled now; it waits for this grid's results itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int num_warps = gridDim.x * kDecWarps;
  UnitCursor cursor;
  int u = blockIdx.x * kDecWarps + warp;
  Unit cu = cursor.seek(a, u);
  if (!cu.ok) return;
  Unit nu = cursor.seek(a, u + num_warps);

  auto load_ids = [&](const Unit& x) -> int {
    if (!x.ok || lane >= x.np) return -1;
    int blk = a.block_table[static_cast<size_t>(x.b) * a.max_blocks + x.p0 + lane];
    if (blk < 0 || blk >= a.num_blocks) {
      report(a.status, KARA_ERR_BAD_BLOCK);
      blk = -1;
    }
    return blk;
  };
  // B fragments of Q^T (column grp = query head g*G + grp when grp < G, else 0): for k-step
  // ks, qb[ks][0] = channels ks*16 + 2*tig + {0,1}, qb[ks][1] = channels ks*16 + 8 + 2*tig + {0,1}
  auto load_q = [&](const Unit& x, uint32_t (&qb)[KS][2]) {
    const bool row_ok = x.ok && grp < G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + (static_cast<size_t>(x.b) * a.Hq + x.g * G + (row_ok ? grp : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qb[ks][0] = row_ok ? qrow[ks * 8 + tig] : 0u;
      qb[ks][1] = row_ok ? qrow[ks * 8 + 4 + tig] : 0u;
    }
  };

  int ids_cu = load_ids(cu), ids_nu = load_ids(nu);
  uint32_t qb[KS][2], qn[KS][2];
  load_q(cu, qb);
  load_q(nu, qn);

  // Stream entries: unit x contributes 2*x.np entries, K pages then V pages.
  int ustart = 0;          // stream index of cu's first entry
  int issued = 0, done = 0;
  uint32_t phase = 0;      // parity bit per stage
  uint32_t pending = 0;    // stages with a load issued and not yet consumed
  volatile int no_abort = 0;
  auto top_up = [&]() {
    const int avail = ustart + 2 * cu.np + (nu.ok ? 2 * nu.np : 0);
    while (issued < done + kStages && issued < avail) {
      const int e = issued - ustart;
      const bool in_cu = e < 2 * cu.np;
      const int e2 = in_cu ? e : e - 2 * cu.np;
      const int npx = in_cu ? cu.np : nu.np;
      const bool is_v = e2 >= npx;
      const int j = is_v ? e2 - npx : e2;
      const int blk = __shfl_sync(0xffffffffu, in_cu ? ids_cu : ids_nu, j & 31);
      const int g = in_cu ? cu.g : nu.g;
      const int st = issued % kStages;
      if (blk >= 0) pending |= 1u << st;
      if (lane == 0 && blk >= 0) {
        uint8_t* dst = my_ring + st * kPage;
        mbar_expect_tx(&my_bars[st], kPage);
        const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
        for (int c = 0; c < NCH; ++c) tma_load_4d(dst + c * kChunkBytes, tm, &my_bars[st], c * 64, g, 0, blk);
      }
      ++issued;
    }
  };
  // Consumes stream entry t: returns the stage's shared address, or 0 when the page was
  // skipped (bad block, reported) or the wait gave up (sets aborted).
  bool aborted = false;
  auto acquire = [&](int t, int blk) -> uint32_t {
    top_up();
    done = t + 1;
    if (blk < 0) return 0u;
    const int st = t % kStages;
    if (!mbar_wait(&my_bars[st], (phase >> st) & 1, &no_abort, a.status)) {
      aborted = true;
      return 0u;
    }
    phase ^= 1u << st;
    pending &= ~(1u << st);
    return ring_u32 + st * kPage;
  };

  while (cu.ok) {
    // ---- K pages: S^T for every page of the unit ----
    float sc[kUnitPages][4];
#pragma unroll
    for (int j = 0; j < kUnitPages; ++j) {
      sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = -INFINITY;
      if (j < cu.np && !aborted) {
        const int blk = __shfl_sync(0xffffffffu, ids_cu, j);
        const uint32_t kst = acquire(ustart + j, blk);
        if (kst != 0u) {
          // two independent accumulator chains (even / odd k-steps), added at the end
          float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            // matrices: (slots 0-7, d lo), (slots 8-15, d lo), (slots 0-7, d hi), (slots 8-15, d hi)
            const int slot = (mtx & 1) * 8 + mrow;
            const int d0 = ks * 16 + (mtx >> 1) * 8;
            uint32_t ka[4];
            ldsm_x4(kst + (d0 >> 6) * kChunkBytes + sw128(slot, (d0 & 63) >> 3), ka);
            mma_16816(acc[ks & 1], ka, qb[ks][0], qb[ks][1]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[0][e] += acc[1][e];
          // acc: (slot grp, heads 2tig, 2tig+1), (slot grp+8, heads 2tig, 2tig+1)
          const int valid = min(16, cu.n - (cu.p0 + j) * 16);
          const bool lo_ok = grp < valid, hi_ok = grp + 8 < valid;
          sc[j][0] = lo_ok ? acc[0][0] * a.cs : -INFINITY;
          sc[j][1] = lo_ok ? acc[0][1] * a.cs : -INFINITY;
          sc[j][2] = hi_ok ? acc[0][2] * a.cs : -INFINITY;
          sc[j][3] = hi_ok ? acc[0][3] * a.cs : -INFINITY;
        }
        __syncwarp();
      }
    }
    if (aborted) break;
    // ---- one exponent base per head over the unit (heads 2tig and 2tig+1) ----
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < kUnitPages; ++j) {
      m0 = fmaxf(m0, fmaxf(sc[j][0], sc[j][2]));
      m1 = fmaxf(m1, fmaxf(sc[j][1], sc[j][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
    }
    const float b0 = m0 == -INFINITY ? 0.f : m0;   // a head with no valid slot: all P = 0
    const float b1 = m1 == -INFINITY ? 0.f : m1;
    float l0 = 0.f, l1 = 0.f;
    uint32_t pb[kUnitPages][2];   // P^T B fragments per page: slots 2tig.. and 8+2tig.., head grp
#pragma unroll
    for (int j = 0; j < kUnitPages; ++j) {
      const float p0 = ex2(sc[j][0] - b0), p1 = ex2(sc[j][1] - b1);
      const float p2 = ex2(sc[j][2] - b0), p3 = ex2(sc[j][3] - b1);
      l0 += p0 + p2;
      l1 += p1 + p3;
      pb[j][0] = movmatrix_trans(pack_bf16(p0, p1));
      pb[j][1] = movmatrix_trans(pack_bf16(p2, p3));
    }
    // ---- V pages: O^T += V^T P^T ----
    float o[KS][4];
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
#pragma unroll
    for (int j = 0; j < kUnitPages; ++j) {
      if (j < cu.np && !aborted) {
        const int blk = __shfl_sync(0xffffffffu, ids_cu, j);
        const uint32_t vst = acquire(ustart + cu.np + j, blk);
        if (vst != 0u) {
          const int valid = min(16, cu.n - (cu.p0 + j) * 16);
          // slots past the context may hold any bits (even NaN); P is 0 there, V is zeroed
          const int s_lo = 2 * tig, s_hi = 8 + 2 * tig;
          const uint32_t mlo = (s_lo < valid ? 0xffffu : 0u) | (s_lo + 1 < valid ? 0xffff0000u : 0u);
          const uint32_t mhi = (s_hi < valid ? 0xffffu : 0u) | (s_hi + 1 < valid ? 0xffff0000u : 0u);
          const bool partial_page = valid < 16;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            // matrices: (slots 0-7, ch lo), (slots 0-7, ch hi), (slots 8-15, ch lo), (slots 8-15, ch hi)
            const int slot = (mtx >> 1) * 8 + mrow;
            const int c0 = mt * 16 + (mtx & 1) * 8;
            uint32_t va[4];
            ldsm_x4_trans(vst + (c0 >> 6) * kChunkBytes + sw128(slot, (c0 & 63) >> 3), va);
            if (partial_page) {
              va[0] &= mlo;
              va[1] &= mlo;
              va[2] &= mhi;
              va[3] &= mhi;
            }
            mma_16816(o[mt], va, pb[j][0], pb[j][1]);
          }
        }
        __syncwarp();
      }
    }
    if (aborted) break;
    // ---- the unit's partial: heads 2tig, 2tig+1 own o[mt][0/2] and o[mt][1/3] ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * tig + e;
      if (h < G) {
        const size_t row = (static_cast<size_t>(cu.b) * a.Hq + cu.g * G + h) * a.S + cu.split;
        float* dst = a.part_o + row * D;
        if (grp == 0) a.part_ml[row] = make_float2(e == 0 ? m0 : m1, e == 0 ? l0 : l1);
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          dst[mt * 16 + grp] = o[mt][e];
          dst[mt * 16 + 8 + grp] = o[mt][2 + e];
        }
      }
    }
    // advance: the next unit becomes current, fetch the one after it
    ustart += 2 * cu.np;
    cu = nu;
    ids_cu = ids_nu;
    if (!cu.ok) break;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qb[ks][0] = qn[ks][0];
      qb[ks][1] = qn[ks][1];
    }
    u += num_warps;
    nu = cursor.seek(a, u + num_warps);
    ids_nu = load_ids(nu);
    load_q(nu, qn);
  }
  if (aborted) {
    // a wait gave up (reported): let this warp's loads still in flight land before exiting
    volatile int give_up = 0;
    for (int st = 0; st < kStages; ++st)
      if ((pending >> st) & 1u) mbar_wait(&my_bars[st], (phase >> st) & 1, &give_up, a.status);
  }
}

// Merge of the split partials of each (sequence, query head): one CTA of kCombWarps warps per
// pair; warp w takes the splits w, w + kCombWarps, ..., lane l owns D/32 consecutive channels,
// and every lane keeps kCombBatch independent loads in flight before it accumulates them. The
// warps' sums meet in shared memory. Launched as a programmatic dependent of the stream kernel:
// its CTAs may start early and wait for the stream kernel's results.
//
// Fused decode step (a.append): the new token at slot n = ctx_len is one more term of the
// softmax, taken from the inputs (s = q . k_new * scale, value v_new); the CTA of the group's
// first query head writes k_new / v_new to slot n of the cache (its block was taken by
// kara_step_begin), and every CTA writes its query to rows n mod W and n mod W + W of the
// window-query ring. The stream kernel, which reads slots [0, n) only, has finished by then.
constexpr int kCombWarps = 8;
constexpr int kCombBatch = 4;

template <int D>
__global__ void __launch_bounds__(32 * kCombWarps)
decode_combine_kernel(const DecodeArgs a, __nv_bfloat16* __restrict__ out) {
  constexpr int V = D / 32;   // channels per lane
  using VecT = typename std::conditional<V == 4, float4, float2>::type;
  __shared__ float red_o[kCombWarps][D];
  __shared__ float red_l[kCombWarps];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int bh = blockIdx.x;
  const int warp = warp_id(), lane = lane_id();
  const int b = bh / a.Hq;
  int n = a.ctx_len[b];
  n = max(0, min(n, a.max_blocks * 16));
  const int splits = (((n + 15) / 16) + kUnitPages - 1) / kUnitPages;
  const float2* ml = a.part_ml + static_cast<size_t>(bh) * a.S;
  const float* po = a.part_o + static_cast<size_t>(bh) * a.S * D + lane * V;
  float mx = -INFINITY;
  for (int s0 = lane; s0 < splits; s0 += 32) mx = fmaxf(mx, ml[s0].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  // the new token's logit (base 2), in every warp; it joins the exponent base
  const int h = bh - b * a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  float s_new = -INFINITY;
  if (a.append) {
    const __nv_bfloat16* qr = a.q + static_cast<size_t>(bh) * D + lane * V;
    const __nv_bfloat16* kr = a.k_new + (static_cast<size_t>(b) * a.Hkv + g) * D + lane * V;
    float dot = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v) dot = fmaf(__bfloat162float(qr[v]), __bfloat162float(kr[v]), dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    s_new = dot * a.cs;
    mx = fmaxf(mx, s_new);
  }
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float lsum = 0.f;
  for (int s0 = warp; s0 < splits; s0 += kCombWarps * kCombBatch) {
    VecT x[kCombBatch];
    float2 mlv[kCombBatch];
#pragma unroll
    for (int i = 0; i < kCombBatch; ++i) {
      const int sp = s0 + i * kCombWarps;
      if (sp < splits) {
        x[i] = *reinterpret_cast<const VecT*>(po + static_cast<size_t>(sp) * D);
        mlv[i] = ml[sp];
      } else {
        mlv[i] = make_float2(-INFINITY, 0.f);
      }
    }
#pragma unroll
    for (int i = 0; i < kCombBatch; ++i) {
      if (mlv[i].x == -INFINITY) continue;
      const float w = ex2(mlv[i].x - mx);
      lsum += w * mlv[i].y;
      const float* xv = reinterpret_cast<const float*>(&x[i]);
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] += w * xv[v];
    }
  }
#pragma unroll
  for (int v = 0; v < V; ++v) red_o[warp][lane * V + v] = acc[v];
  if (lane == 0) red_l[warp] = lsum;
  __syncthreads();
  if (warp == 0) {
    float l = 0.f, r[V];
#pragma unroll
    for (int v = 0; v < V; ++v) r[v] = 0.f;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) {
      l += red_l[w];
#pragma unroll
      for (int v = 0; v < V; ++v) r[v] += red_o[w][lane * V + v];
    }
    if (a.append) {
      const float w = ex2(s_new - mx);
      const __nv_bfloat16* vr = a.v_new + (static_cast<size_t>(b) * a.Hkv + g) * D + lane * V;
      l += w;
#pragma unroll
      for (int v = 0; v < V; ++v) r[v] = fmaf(w, __bfloat162float(vr[v]), r[v]);
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* dst = out + static_cast<size_t>(bh) * D + lane * V;
#pragma unroll
    for (int v = 0; v < V; v += 2)
      *reinterpret_cast<__nv_bfloat162*>(dst + v) = __floats2bfloat162_rn(r[v] * inv, r[v + 1] * inv);
  } else if (warp == 1 && a.append) {
    // the new token into the cache (one CTA per KV head) and its query into the ring
    const int n_raw = a.ctx_len[b];
    if (n_raw < 0 || n_raw >= a.max_blocks * 16) {
      if (lane == 0) report(a.status, KARA_ERR_INVALID_ARG);
    } else {
      if (h % (a.Hq / a.Hkv) == 0) {
        const int blk = a.block_table[static_cast<size_t>(b) * a.max_blocks + n_raw / 16];
        if (blk < 0 || blk >= a.num_blocks) {
          if (lane == 0) report(a.status, KARA_ERR_BAD_BLOCK);
        } else {
          const size_t row = ((static_cast<size_t>(blk) * 16 + n_raw % 16) * a.Hkv + g) * D + lane * V;
          const size_t src = (static_cast<size_t>(b) * a.Hkv + g) * D + lane * V;
#pragma unroll
          for (int v = 0; v < V; ++v) {
            a.k_dst[row + v] = a.k_new[src + v];
            a.v_dst[row + v] = a.v_new[src + v];
          }
        }
      }
      if (a.q_ring != nullptr) {
        const int p = n_raw % a.ring_w;
        const __nv_bfloat16* qr = a.q + static_cast<size_t>(bh) * D + lane * V;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          __nv_bfloat16* dq = a.q_ring +
              ((static_cast<size_t>(b) * 2 * a.ring_w + p + e * a.ring_w) * a.Hq + h) * D + lane * V;
#pragma unroll
          for (int v = 0; v < V; ++v) dq[v] = qr[v];
        }
      }
    }
  }
}

template <int D, int G, bool DEEP>
kara_status launch_dg(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, void* out,
                      cudaStream_t stream) {
  constexpr size_t smem = stream_smem_bytes<D, DEEP>();
  static std::atomic<int> per_sm[kMaxDevices];   // resident CTAs per SM, queried once per device
  const int dev = device_slot();
  if (dev < 0) {
    set_last_error("paged_decode_attn", "no usable current CUDA device");
    return KARA_ERR_CUDA;
  }
  if (per_sm[dev].load() == 0) {
    cudaFuncSetAttribute(decode_stream_kernel<D, G, DEEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_stream_kernel<D, G, DEEP>, kDecThreads, smem);
    per_sm[dev].store(n > 0 ? n : 1);
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  launch_pdl(decode_stream_kernel<D, G, DEEP>, dim3(per_sm[dev].load() * sms), dim3(kDecThreads), smem,
             stream, tk, tv, a);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Hq);
  cfg.blockDim = dim3(32 * kCombWarps);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch(cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, a,
                                  static_cast<__nv_bfloat16*>(out)));
  return check_launch(__func__);
}

// Ring shape per instantiation. At 128 registers (4 CTAs per SM) the d = 128 stream spills
// 4-12 bytes for G <= 6 (ptxas); those run 3 CTAs per SM with 4-page rings, which measured 8 %
// faster at G = 4 with 4 and with 8 KV heads. G = 7 and 8 fit 128 registers without spills and
// run 4 CTAs per SM with 3-page rings, 0.8-0.9 % faster with 4 and with 8 KV heads. d = 64 fits
// either way (at most 125 registers) and keeps the shallow rings.
template <int D, int G>
constexpr bool deep_ring() { return D == 128 && G <= 6; }

template <int D>
kara_status launch_d(const DecodeArgs& a, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                     void* out, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_dg<D, 1, deep_ring<D, 1>()>(a, tk, tv, out, stream);
    case 2: return launch_dg<D, 2, deep_ring<D, 2>()>(a, tk, tv, out, stream);
    case 3: return launch_dg<D, 3, deep_ring<D, 3>()>(a, tk, tv, out, stream);
    case 4: return launch_dg<D, 4, deep_ring<D, 4>()>(a, tk, tv, out, stream);
    case 5: return launch_dg<D, 5, deep_ring<D, 5>()>(a, tk, tv, out, stream);
    case 6: return launch_dg<D, 6, deep_ring<D, 6>()>(a, tk, tv, out, stream);
    case 7: return launch_dg<D, 7, deep_ring<D, 7>()>(a, tk, tv, out, stream);
    case 8: return launch_dg<D, 8, deep_ring<D, 8>()>(a, tk, tv, out, stream);
    default: return KARA_ERR_UNSUPPORTED;
  }
}

}  // namespace

int decode_num_splits(int max_blocks) { return (max_blocks + kUnitPages - 1) / kUnitPages; }

size_t decode_workspace_bytes(int B, int Hq, int D, int max_blocks) {
  return static_cast<size_t>(B) * Hq * decode_num_splits(max_blocks) * (D + 2) * sizeof(float);
}

kara_status launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
  if (L.B == 0) return KARA_OK;
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(L.q);
  a.k = static_cast<const __nv_bfloat16*>(L.k_cache);
  a.v = static_cast<const __nv_bfloat16*>(L.v_cache);
  a.block_table = L.block_table;
  a.ctx_len = L.ctx_len;
  // workspace: o rows [B, Hq, S, D] first, then (m, l) pairs [B, Hq, S]
  a.S = decode_num_splits(L.max_blocks);
  a.part_o = L.partial;
  a.part_ml = reinterpret_cast<float2*>(L.partial + static_cast<size_t>(L.B) * L.Hq * a.S * L.D);
  a.status = L.status;
  a.B = L.B;
  a.Hq = L.Hq;
  a.Hkv = L.Hkv;
  a.max_blocks = L.max_blocks;
  a.num_blocks = L.num_blocks;
  a.cs = L.scale * 1.4426950408889634f;
  a.append = L.k_new != nullptr ? 1 : 0;
  a.k_new = static_cast<const __nv_bfloat16*>(L.k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(L.v_new);
  a.k_dst = static_cast<__nv_bfloat16*>(const_cast<void*>(L.k_cache));
  a.v_dst = static_cast<__nv_bfloat16*>(const_cast<void*>(L.v_cache));
  a.q_ring = static_cast<__nv_bfloat16*>(L.q_ring);
  a.ring_w = L.ring_w;
  const int G = L.Hq / L.Hkv;
  // paged pools as 4-D maps {d, Hkv, 16 slots, blocks}; box = one page of one KV head, 64
  // channels wide, 128-byte swizzle (the same map shape the scoring kernels use)
  const uint64_t dims[4] = {static_cast<uint64_t>(L.D), static_cast<uint64_t>(L.Hkv), 16,
                            static_cast<uint64_t>(L.num_blocks)};
  const uint64_t strides[3] = {static_cast<uint64_t>(L.D) * 2, static_cast<uint64_t>(L.Hkv) * L.D * 2,
                               static_cast<uint64_t>(16) * L.Hkv * L.D * 2};
  CUtensorMap tk, tv;
  if (!make_bf16_map_4d(&tk, L.k_cache, dims, strides, 16) ||
      !make_bf16_map_4d(&tv, L.v_cache, dims, strides, 16))
    return KARA_ERR_CUDA;
  if (L.D == 128) return launch_d<128>(a, G, tk, tv, L.out, stream);
  if (L.D == 64) return launch_d<64>(a, G, tk, tv, L.out, stream);
  return KARA_ERR_UNSUPPORTED;
}

}  // namespace kara
