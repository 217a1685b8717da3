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
// splits of each (sequence, query head). Per page a warp assigns two lanes to each of the 16
// slots (half of d each) for q.k, then one lane per 4 channels of d for p.v; K rows are read
// with 16-byte loads, V rows with 8-byte loads, both coalesced within a row.
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

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const DecodeArgs a) {
  constexpr int kHalf = D / 2;          // channels per lane in q.k
  constexpr int kVec = kHalf / 8;       // 16-byte K loads per lane
  constexpr int kE4 = kHalf / 4;        // float4 groups per half
  constexpr int kCh = D / 32;           // channels per lane in p.v (4 or 2)
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

  __shared__ __align__(16) float q_s[G][kE4][2][4];          // pre-scaled q, half-interleaved
  __shared__ __align__(16) float p_s[kDecWarps][16][8];       // page probabilities
  __shared__ float red_m[kDecWarps][G], red_l[kDecWarps][G];
  __shared__ __align__(16) float red_o[kDecWarps][G][D];

  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int h = i / D, c = i % D;
    const float qv = __bfloat162float(a.q[(static_cast<size_t>(b) * a.Hq + g * G + h) * D + c]);
    const int half = c / kHalf, e = c % kHalf;
    q_s[h][e / 4][half][e % 4] = qv * a.cs;
  }
  __syncthreads();

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
  const size_t row_stride = static_cast<size_t>(a.Hkv) * D;   // elements between slots
  const int32_t* tab = a.block_table + static_cast<size_t>(b) * a.max_blocks;

  for (int p = p_begin + warp; p < p_end; p += kDecWarps) {
    const int blk = tab[p];
    if (blk < 0 || blk >= a.num_blocks) {
      if (lane == 0) report(a.status, KARA_ERR_BAD_BLOCK);
      continue;
    }
    const int valid = min(16, n - p * 16);
    const __nv_bfloat16* kpage = a.k + (static_cast<size_t>(blk) * 16) * row_stride + g * D;
    const __nv_bfloat16* vpage = a.v + (static_cast<size_t>(blk) * 16) * row_stride + g * D;
    // issue the loads of the page: K (this lane's slot, half of d) and V (all 16 slots, kCh
    // channels of this lane)
    uint4 kr[kVec];
    const uint4* kp4 = reinterpret_cast<const uint4*>(kpage + slot * row_stride + half * kHalf);
#pragma unroll
    for (int i = 0; i < kVec; ++i) kr[i] = kp4[i];
    uint32_t vr[16][kCh / 2];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      const __nv_bfloat16* vrow = vpage + s * row_stride + lane * kCh;
      if (s < valid) {
        if constexpr (kCh == 4) {
          const uint2 t = *reinterpret_cast<const uint2*>(vrow);
          vr[s][0] = t.x;
          vr[s][1] = t.y;
        } else {
          vr[s][0] = *reinterpret_cast<const uint32_t*>(vrow);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kCh / 2; ++c) vr[s][c] = 0u;
      }
    }
    // q . k for this lane's slot and half of d, as pairs of partial sums
    float2 dot2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) dot2[h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const float2 k01 = bf16x2_to_f2(kr[i].x), k23 = bf16x2_to_f2(kr[i].y);
      const float2 k45 = bf16x2_to_f2(kr[i].z), k67 = bf16x2_to_f2(kr[i].w);
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
    // p . v
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      float2 vf[kCh / 2];
#pragma unroll
      for (int c = 0; c < kCh / 2; ++c) vf[c] = bf16x2_to_f2(vr[s][c]);
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

  // merge the four warps of the CTA
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) { red_m[warp][h] = m[h]; red_l[warp][h] = l[h]; }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < kCh / 2; ++c) {
      red_o[warp][h][lane * kCh + 2 * c] = acc[h][c].x;
      red_o[warp][h][lane * kCh + 2 * c + 1] = acc[h][c].y;
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
        val += wt * (c == 1 ? red_l[w][h] : red_o[w][h][c - 2]);
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
kara_status launch_dg(const DecodeArgs& a, void* out, cudaStream_t stream) {
  dim3 grid(a.S, a.Hkv, a.B);
  decode_split_kernel<D, G><<<grid, kDecThreads, 0, stream>>>(a);
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, stream>>>(a, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError() == cudaSuccess ? KARA_OK : KARA_ERR_CUDA;
}

template <int D>
kara_status launch_d(const DecodeArgs& a, int G, void* out, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_dg<D, 1>(a, out, stream);
    case 2: return launch_dg<D, 2>(a, out, stream);
    case 3: return launch_dg<D, 3>(a, out, stream);
    case 4: return launch_dg<D, 4>(a, out, stream);
    case 5: return launch_dg<D, 5>(a, out, stream);
    case 6: return launch_dg<D, 6>(a, out, stream);
    case 7: return launch_dg<D, 7>(a, out, stream);
    case 8: return launch_dg<D, 8>(a, out, stream);
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
  if (L.D == 128) return launch_d<128>(a, G, L.out, stream);
  if (L.D == 64) return launch_d<64>(a, G, L.out, stream);
  return KARA_ERR_UNSUPPORTED;
}

}  // namespace kara
