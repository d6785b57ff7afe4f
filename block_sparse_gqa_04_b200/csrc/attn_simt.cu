// Main branch on CUDA cores, KV-outer: one CTA per 128-row tile of one block's
// query list ("MiniMax 稀疏注意力" (hyper.ai), section 引言: the FlashAttention
// loop order is swapped so each KV block is read once for the queries that
// chose it).  Each (query, head, slot) row is one query head against one block:
// the softmax over that block's visible tokens is complete inside the tile, so
// the kernel writes the normalised partial output and its base-2 log-normaliser
// and the combine kernel merges the slots.  Used for fp32 problems and for the
// shapes the tensor-core kernel does not cover.  With fp8 (e4m3) q and k the
// scores are formed from those values (widened exactly to fp32); v stays bf16.
#include "common.cuh"
#include "internal.h"

namespace msa {

// Finds the list that holds tile `tile`: the last L with tile_off[L] <= tile.
__device__ __forceinline__ long long find_list(const int32_t* __restrict__ tile_off,
                                               long long nlists, int tile) {
  long long lo = 0, hi = nlists;  // invariant: tile_off[lo] <= tile < tile_off[hi]
  while (hi - lo > 1) {
    long long mid = (lo + hi) >> 1;
    if (tile_off[mid] <= tile) lo = mid; else hi = mid;
  }
  return lo;
}

// TQ: element type of q and k (the scores q . k), TV: of v.
template <typename TQ, typename TV, typename PT, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(Problem P, const TQ* __restrict__ q,
                                                        const TQ* __restrict__ k,
                                                        const TV* __restrict__ v, Lists L,
                                                        PT* __restrict__ part_o,
                                                        float* __restrict__ part_lse) {
  constexpr int EPL = D / 32;  // elements per lane
  extern __shared__ unsigned char smem_raw[];
  TQ* ks = reinterpret_cast<TQ*>(smem_raw);                        // [Bk][D]
  TV* vs = reinterpret_cast<TV*>(smem_raw + 128 * D * sizeof(TQ));  // [Bk][D]
  float* sc = reinterpret_cast<float*>(vs + 128 * D);              // [4 warps][Bk]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int total_tiles = L.tile_off[P.nlists];
  const float scale_log2 = P.scale * 1.4426950408889634f;
  for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
    const long long lid = find_list(L.tile_off, P.nlists, tile);
    const int c = int(lid % P.nblk);
    const long long rest = lid / P.nblk;  // (b * Hkv + g) * nqc + qc
    const int g = int((rest / P.nqc) % P.Hkv);
    const int b = int(rest / ((long long)P.nqc * P.Hkv));
    const int e0 = L.list_off[lid] + (tile - L.tile_off[lid]) * P.qpt;
    const int e1 = min(e0 + P.qpt, L.list_off[lid + 1]);
    const long long j0 = (long long)c * P.Bk;
    const int nkeys = (int)min((long long)P.Bk, (long long)P.Skv - j0);
    __syncthreads();  // previous tile done with ks / vs
    for (int e = threadIdx.x; e < nkeys * D; e += blockDim.x) {
      const int j = e / D, d = e % D;
      const long long src = ((block_row(P, b, c) + j) * P.Hkv + g) * D + d;
      ks[e] = k[src];
      vs[e] = v[src];
    }
    __syncthreads();
    float* s = sc + warp * 128;
    const int rows = (e1 - e0) * P.G;
    for (int ri = warp; ri < rows; ri += 4) {
      const int packed = L.entries[e0 + ri / P.G];
      const int h = g * P.G + ri % P.G;
      const int r = packed >> 5;
      const long long t = P.q_pos0 + r % P.Sq;
      const int jn = (int)min((long long)nkeys, t - j0 + 1);
      float qv[EPL];
      load_vec<TQ, EPL>(q + ((long long)r * P.Hq + h) * D + lane * EPL, qv);
      float m = -INFINITY;
      for (int j = 0; j < jn; ++j) {
        float kv[EPL];
        load_vec<TQ, EPL>(ks + j * D + lane * EPL, kv);
        float acc = 0.f;
#pragma unroll
        for (int x = 0; x < EPL; ++x) acc = fmaf(qv[x], kv[x], acc);
        acc = warp_sum_f32(acc) * scale_log2;
        if (lane == 0) s[j] = acc;
        m = fmaxf(m, acc);
      }
      __syncwarp();
      float o[EPL];
#pragma unroll
      for (int x = 0; x < EPL; ++x) o[x] = 0.f;
      float l = 0.f;
      for (int j = 0; j < jn; ++j) {
        const float p = exp2f(s[j] - m);
        l += p;
        float vv[EPL];
        load_vec<TV, EPL>(vs + j * D + lane * EPL, vv);
#pragma unroll
        for (int x = 0; x < EPL; ++x) o[x] = fmaf(p, vv[x], o[x]);
      }
      __syncwarp();
      const float inv = 1.f / l;
      const long long pidx = (long long)(e0 + ri / P.G) * P.G + ri % P.G;
      PT* dst = part_o + pidx * D + lane * EPL;
#pragma unroll
      for (int x = 0; x < EPL; ++x) dst[x] = from_f32<PT>(o[x] * inv);
      if (lane == 0) part_lse[pidx] = m + log2f(l);
    }
  }
}

template <typename TQ, typename TV, typename PT, int D>
static cudaError_t launch_t(const Problem& P, const void* q, const void* k, const void* v,
                            const Lists& L, const Partials& part, cudaStream_t s) {
  size_t smem = 128 * D * (sizeof(TQ) + sizeof(TV)) + 4 * 128 * sizeof(float);
  auto kern = attn_simt_kernel<TQ, TV, PT, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  kern<<<148 * 4, 128, smem, s>>>(P, (const TQ*)q, (const TQ*)k, (const TV*)v, L,
                                  (PT*)part.o, part.lse2);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const Problem& P, const void* q, const void* k, const void* v,
                             const Lists& L, const Partials& part, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  using fp8 = __nv_fp8_e4m3;
  if (P.f32) {
    return P.D == 64 ? launch_t<float, float, float, 64>(P, q, k, v, L, part, s)
                     : launch_t<float, float, float, 128>(P, q, k, v, L, part, s);
  }
  if (P.qk8) {
    return P.D == 64 ? launch_t<fp8, bf16, bf16, 64>(P, q, k, v, L, part, s)
                     : launch_t<fp8, bf16, bf16, 128>(P, q, k, v, L, part, s);
  }
  return P.D == 64 ? launch_t<bf16, bf16, bf16, 64>(P, q, k, v, L, part, s)
                   : launch_t<bf16, bf16, bf16, 128>(P, q, k, v, L, part, s);
}

}  // namespace msa
