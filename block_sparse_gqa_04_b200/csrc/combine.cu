// Merge of the per-slot partial softmax states of one (query row, head).
//
// The KV-outer kernels finish the softmax of each (row, head, slot) over one
// block and store o_s (normalised) and lse_s = log2 of its normaliser, at the
// entry position the block -> query lists gave that (group, row, slot).  The
// exact softmax over the union of the slots' tokens is
//     O = sum_s w_s o_s,   w_s = 2^(lse_s - M) / sum_u 2^(lse_u - M),
// with M = max_s lse_s, and its natural-log normaliser is (M + log2 sum) ln 2.
// One warp per (row, head); lane s reads slot s's lse, each lane owns D/32
// output elements.
#include "common.cuh"
#include "internal.h"

namespace msa {

template <typename PT, typename OT, int D>
__global__ void __launch_bounds__(256) combine_kernel(Problem P, const int32_t* __restrict__ pos,
                                                      const PT* __restrict__ part_o,
                                                      const float* __restrict__ part_lse,
                                                      OT* __restrict__ out,
                                                      float* __restrict__ lse_out) {
  constexpr int EPL = D / 32;
  const int lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (long long)P.T * P.Hq) return;
  const int r = int(wid / P.Hq), h = int(wid % P.Hq);
  const int g = h / P.G, hh = h % P.G;
  // lane s < K looks after slot s: its partial sits at entry position pos[g, r, s]
  long long prow = -1;
  float ls = -INFINITY;
  if (lane < P.K) {
    const int e = pos[((long long)g * P.T + r) * P.K + lane];
    if (e >= 0) {
      prow = (long long)e * P.G + hh;
      ls = part_lse[prow];
    }
  }
  const float M = warp_max_f32(ls);
  float o[EPL];
#pragma unroll
  for (int x = 0; x < EPL; ++x) o[x] = 0.f;
  OT* dst = out + ((long long)r * P.Hq + h) * D + lane * EPL;
  if (M == -INFINITY) {  // no valid slot
#pragma unroll
    for (int x = 0; x < EPL; ++x) dst[x] = from_f32<OT>(0.f);
    if (lse_out && lane == 0) lse_out[(long long)r * P.Hq + h] = -INFINITY;
    return;
  }
  const float w = ls == -INFINITY ? 0.f : exp2f(ls - M);
  const float sum = warp_sum_f32(w);
  const float inv = 1.f / sum;
  unsigned valid = __ballot_sync(MSA_FULL_MASK, w > 0.f);
  while (valid) {
    const int s = __ffs(valid) - 1;
    valid &= valid - 1;
    const float ws = __shfl_sync(MSA_FULL_MASK, w, s) * inv;
    const long long ps = __shfl_sync(MSA_FULL_MASK, prow, s);
    float pv[EPL];
    load_vec<PT, EPL>(part_o + ps * D + lane * EPL, pv);
#pragma unroll
    for (int x = 0; x < EPL; ++x) o[x] = fmaf(ws, pv[x], o[x]);
  }
#pragma unroll
  for (int x = 0; x < EPL; ++x) dst[x] = from_f32<OT>(o[x]);
  if (lse_out && lane == 0)
    lse_out[(long long)r * P.Hq + h] = (M + log2f(sum)) * 0.6931471805599453f;
}

template <typename T, int D>
static cudaError_t launch_t(const Problem& P, const int32_t* pos, const Partials& part,
                            void* out, float* lse, cudaStream_t s) {
  long long warps = (long long)P.T * P.Hq;
  long long blocks = (warps + 7) / 8;
  combine_kernel<T, T, D><<<unsigned(blocks), 256, 0, s>>>(P, pos, (const T*)part.o,
                                                           part.lse2, (T*)out, lse);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Problem& P, const int32_t* pos, const Partials& part,
                           void* out, float* lse, cudaStream_t s) {
  if ((long long)P.T * P.Hq == 0) return cudaSuccess;
  if (P.f32) return P.D == 64 ? launch_t<float, 64>(P, pos, part, out, lse, s)
                              : launch_t<float, 128>(P, pos, part, out, lse, s);
  return P.D == 64 ? launch_t<__nv_bfloat16, 64>(P, pos, part, out, lse, s)
                   : launch_t<__nv_bfloat16, 128>(P, pos, part, out, lse, s);
}

}  // namespace msa
