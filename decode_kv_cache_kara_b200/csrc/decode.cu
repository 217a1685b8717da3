// Paged grouped-query decode attention over the (compressed) cache, split-KV.
//
// out[b][h] = sum_t softmax_t(q_bh . k_t * scale) v_t over the slots [0, ctx_len[b]) read
// through the block table ("Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache
// Compression", English abstract: the kept KV pairs serve subsequent decoding; the method is
// adapted to PagedAttention).
//
// HBM-bound: every K and V row of a KV head is loaded once for all G query heads of its group.
// Grid = (split, KV head, sequence); a split covers 16 pages; each of the 4 warps walks its
// pages with its own online softmax (base 2, scale folded into q), and the warps merge in
// shared memory into one split partial (m, l, unnormalised o). A second kernel merges the
// splits of each (sequence, query head). Pages reach shared memory by TMA (one 16-row box of
// one KV head per 64 channels, 128-byte swizzle) through a 3-stage ring per warp, so that
// each SM keeps many pages in flight. Per page a warp assigns two lanes to each of the 16
// slots (half of d each) for q.k, then one lane per 4 channels of d for p.v; the swizzle
// keeps both read patterns free of bank conflicts.
#include <cuda.h>

#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace kara {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = 4;
constexpr int kPagesPerSplit = 16;

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* block_table;
  const int32_t* ctx_len;
  float* partial;      // [B, Hq, S, D + 2]: m, l, o[D]
  int32_t* status;
  int B, Hq, Hkv, max_blocks, num_blocks, S;
  float cs;            // scale * log2(e)
};

template <int D>
__host__ __device__ constexpr int page_bytes() { return 16 * D * 2; }   // one page, one KV head
constexpr int kStages = 3;                                  // TMA page ring depth per warp

template <int D, int G>
constexpr size_t split_smem_bytes() {
  // [warp][stage]{K page, V page} (1024-aligned); the warp merge reuses this space
  return 1024 + static_cast<size_t>(kDecWarps) * kStages * 2 * page_bytes<D>() + 64 * kDecWarps;
}

// Byte offset of 16-byte granule `gi` of row `r` in a 128-byte-swizzled 16-row box.
__device__ __forceinline__ uint32_t sw128(int r, int gi) {
  return static_cast<uint32_t>(r * 128 + ((gi ^ (r & 7)) << 4));
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecodeArgs a) {
  constexpr int NCH = D / 64;                 // 64-channel chunks per row
  constexpr int kHalf = D / 2;                // channels per lane in q.k
  constexpr int kE4 = kHalf / 4;              // float4 groups per half
  constexpr int kCh = D / 32;                 // channels per lane in p.v (4 or 2)
  constexpr uint32_t kPage = page_bytes<D>();
  constexpr uint32_t kChunkBytes = 16 * 128;  // one 64-channel chunk of a page
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();

  int n = a.ctx_len[b];
  if (n > a.max_blocks * 16) {
    if (threadIdx.x == 0 && split == 0 && g == 0) report(a.status, KARA_ERR_INVALID_ARG);
    n = a.max_blocks * 16;
  }
  const int pages = (n + 15) / 16;
  const int p_begin = split * kPagesPerSplit;
  if (p_begin >= pages) return;
  const int p_end = min(pages, p_begin + kPagesPerSplit);

  extern __shared__ __align__(1024) uint8_t dsm[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* my_ring = ring + static_cast<size_t>(warp) * kStages * 2 * kPage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kDecWarps * kStages * 2 * kPage);
  uint64_t* my_bars = bars + warp * kStages;
  __shared__ __align__(16) float q_s[G][kE4][2][4];          // pre-scaled q, half-interleaved
  __shared__ __align__(16) float p_s[kDecWarps][16][8];       // page probabilities
  __shared__ float red_m[kDecWarps][G], red_l[kDecWarps][G];
  float* red_o = reinterpret_cast<float*>(ring);              // [warp][G][D], after the loop

  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&my_bars[st], 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int h = i / D, c = i % D;
    const float qv = __bfloat162float(a.q[(static_cast<size_t>(b) * a.Hq + g * G + h) * D + c]);
    const int half = c / kHalf, e = c % kHalf;
    q_s[h][e / 4][half][e % 4] = qv * a.cs;
  }
  __syncthreads();

  // this warp's pages: p_begin + warp + 4k; lane k holds the block id of its k-th page
  const int32_t* tab = a.block_table + static_cast<size_t>(b) * a.max_blocks;
  const int my_pages = (p_end - p_begin - warp + kDecWarps - 1) / kDecWarps;
  int my_blk = 0;
  if (lane < my_pages) {
    my_blk = tab[p_begin + warp + kDecWarps * lane];
    if (my_blk < 0 || my_blk >= a.num_blocks) {
      report(a.status, KARA_ERR_BAD_BLOCK);
      my_blk = -1;
    }
  }
  auto issue = [&](int k) {          // lane 0: page k of this warp into stage k % kStages
    const int blk = __shfl_sync(0xffffffffu, my_blk, k);
    if (lane == 0 && blk >= 0) {
      uint8_t* st = my_ring + (k % kStages) * 2 * kPage;
      uint64_t* bar = &my_bars[k % kStages];
      mbar_expect_tx(bar, 2 * kPage);
      for (int c = 0; c < NCH; ++c) {
        tma_load_4d(st + c * kChunkBytes, &tm_k, bar, c * 64, g, 0, blk);
        tma_load_4d(st + kPage + c * kChunkBytes, &tm_v, bar, c * 64, g, 0, blk);
      }
    }
  };
  for (int k = 0; k < min(kStages, my_pages); ++k) issue(k);

  float m[G], l[G];
  float2 acc[G][kCh / 2];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int c = 0; c < kCh / 2; ++c) acc[h][c] = make_float2(0.f, 0.f);
  }
  const int slot = lane >> 1, half = lane & 1;
  uint32_t phase_bits = 0;            // parity per stage
  volatile int no_abort = 0;

  for (int k = 0; k < my_pages; ++k) {
    const int p = p_begin + warp + kDecWarps * k;
    const int blk = __shfl_sync(0xffffffffu, my_blk, k);
    const int st = k % kStages;
    if (blk >= 0) {                                 // a bad block id was reported; page skipped
    const bool ok = mbar_wait(&my_bars[st], (phase_bits >> st) & 1, &no_abort, a.status);
    phase_bits ^= 1u << st;
    if (!ok) break;
    const int valid = min(16, n - p * 16);
    const uint8_t* kst = my_ring + st * 2 * kPage;
    const uint8_t* vst = kst + kPage;
    // q . k: this lane's slot, half of d (granules of chunk `half` for d = 128, the half of
    // chunk 0's granules for d = 64)
    float2 dot2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) dot2[h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kHalf / 8; ++i) {
      const int chunk = NCH == 2 ? half : 0;
      const int gi = NCH == 2 ? i : half * 4 + i;
      const uint4 kr = *reinterpret_cast<const uint4*>(kst + chunk * kChunkBytes + sw128(slot, gi));
      const float2 k01 = bf16x2_to_f2(kr.x), k23 = bf16x2_to_f2(kr.y);
      const float2 k45 = bf16x2_to_f2(kr.z), k67 = bf16x2_to_f2(kr.w);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 qa = *reinterpret_cast<const float4*>(&q_s[h][2 * i][half][0]);
        const float4 qb = *reinterpret_cast<const float4*>(&q_s[h][2 * i + 1][half][0]);
        float2 d = dot2[h];
        d = ffma2(k01, make_float2(qa.x, qa.y), d);
        d = ffma2(k23, make_float2(qa.z, qa.w), d);
        d = ffma2(k45, make_float2(qb.x, qb.y), d);
        d = ffma2(k67, make_float2(qb.z, qb.w), d);
        dot2[h] = d;
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float d = dot2[h].x + dot2[h].y;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      if (slot >= valid) d = -INFINITY;
      float pm = d;
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, off));
      const float m_new = fmaxf(m[h], pm);
      const float corr = ex2(m[h] - m_new);
      const float pr = ex2(d - m_new);
      float ps = pr;
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[h] = l[h] * corr + ps;
      m[h] = m_new;
#pragma unroll
      for (int c = 0; c < kCh / 2; ++c) acc[h][c] = fmul2(acc[h][c], make_float2(corr, corr));
      if (half == 0) p_s[warp][slot][h] = pr;
    }
    __syncwarp();
    // p . v: channels [kCh*lane, kCh*lane + kCh) of every valid slot
    const int c0 = kCh * lane;
    const int vchunk = c0 / 64, vgi = (c0 % 64) / 8, vsub = ((c0 % 64) % 8) * 2;
    for (int s = 0; s < valid; ++s) {
      const uint8_t* vrow = vst + vchunk * kChunkBytes + sw128(s, vgi) + vsub;
      float2 vf[kCh / 2];
      if constexpr (kCh == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(vrow);
        vf[0] = bf16x2_to_f2(t.x);
        vf[1] = bf16x2_to_f2(t.y);
      } else {
        vf[0] = bf16x2_to_f2(*reinterpret_cast<const uint32_t*>(vrow));
      }
      const float4 p0 = *reinterpret_cast<const float4*>(&p_s[warp][s][0]);
      const float4 p1 = *reinterpret_cast<const float4*>(&p_s[warp][s][4]);
      const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 pp = make_float2(pv[h], pv[h]);
#pragma unroll
        for (int c = 0; c < kCh / 2; ++c) acc[h][c] = ffma2(pp, vf[c], acc[h][c]);
      }
    }
    __syncwarp();
    }
    // stage st is free again: refill it with page k + kStages
    if (k + kStages < my_pages) {
      fence_proxy_async();
      issue(k + kStages);
    }
  }
  __syncthreads();    // every warp is done with the ring: reuse it for the merge

  // merge the four warps of the CTA
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) { red_m[warp][h] = m[h]; red_l[warp][h] = l[h]; }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < kCh / 2; ++c) {
      red_o[(warp * G + h) * D + lane * kCh + 2 * c] = acc[h][c].x;
      red_o[(warp * G + h) * D + lane * kCh + 2 * c + 1] = acc[h][c].y;
    }
  __syncthreads();
  for (int i = threadIdx.x; i < G * (D + 2); i += kDecThreads) {
    const int h = i / (D + 2), c = i % (D + 2);
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) mx = fmaxf(mx, red_m[w][h]);
    float val = 0.f;
    if (c == 0) {
      val = mx;
    } else {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = (red_m[w][h] == -INFINITY) ? 0.f : ex2(red_m[w][h] - mx);
        val += wt * (c == 1 ? red_l[w][h] : red_o[(w * G + h) * D + c - 2]);
      }
    }
    a.partial[((static_cast<size_t>(b) * a.Hq + g * G + h) * a.S + split) * (D + 2) + c] = val;
  }
}

template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const DecodeArgs a, __nv_bfloat16* __restrict__ out) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hq;
  int n = a.ctx_len[b];
  n = min(n, a.max_blocks * 16);
  const int splits = (((n + 15) / 16) + kPagesPerSplit - 1) / kPagesPerSplit;
  const float* part = a.partial + static_cast<size_t>(bh) * a.S * (D + 2);
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part[s * (D + 2)]);
  float lsum = 0.f, o = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = part[s * (D + 2)];
    if (ms == -INFINITY) continue;
    const float w = ex2(ms - mx);
    lsum += w * part[s * (D + 2) + 1];
    o += w * part[s * (D + 2) + 2 + threadIdx.x];
  }
  const float res = lsum > 0.f ? o / lsum : 0.f;
  out[static_cast<size_t>(bh) * D + threadIdx.x] = __float2bfloat16_rn(res);
}

template <int D, int G>
kara_status launch_dg(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, void* out,
                      cudaStream_t stream) {
  dim3 grid(a.S, a.Hkv, a.B);
  constexpr size_t smem = split_smem_bytes<D, G>();
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(decode_split_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    attr = true;
  }
  decode_split_kernel<D, G><<<grid, kDecThreads, smem, stream>>>(tk, tv, a);
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, stream>>>(a, static_cast<__nv_bfloat16*>(out));
  return check_launch(__func__);
}

template <int D>
kara_status launch_d(const DecodeArgs& a, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                     void* out, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_dg<D, 1>(a, tk, tv, out, stream);
    case 2: return launch_dg<D, 2>(a, tk, tv, out, stream);
    case 3: return launch_dg<D, 3>(a, tk, tv, out, stream);
    case 4: return launch_dg<D, 4>(a, tk, tv, out, stream);
    case 5: return launch_dg<D, 5>(a, tk, tv, out, stream);
    case 6: return launch_dg<D, 6>(a, tk, tv, out, stream);
    case 7: return launch_dg<D, 7>(a, tk, tv, out, stream);
    case 8: return launch_dg<D, 8>(a, tk, tv, out, stream);
    default: return KARA_ERR_UNSUPPORTED;
  }
}

}  // namespace

int decode_num_splits(int max_blocks) { return (max_blocks + kPagesPerSplit - 1) / kPagesPerSplit; }

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
  a.partial = L.partial;
  a.status = L.status;
  a.B = L.B;
  a.Hq = L.Hq;
  a.Hkv = L.Hkv;
  a.max_blocks = L.max_blocks;
  a.num_blocks = L.num_blocks;
  a.S = decode_num_splits(L.max_blocks);
  a.cs = L.scale * 1.4426950408889634f;
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
