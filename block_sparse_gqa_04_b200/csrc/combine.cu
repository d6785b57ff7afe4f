// Merge of the per-slot partial softmax states of one (query row, head).
//
// The KV-outer kernels finish the softmax of each (row, head, slot) over one
// block and store o_s (normalised) and lse_s = log2 of its normaliser, at the
// entry position the block -> query lists gave that (group, row, slot).  The
// exact softmax over the union of the slots' tokens is
//     O = sum_s w_s o_s,   w_s = 2^(lse_s - M) / sum_u 2^(lse_u - M),
// with M = max_s lse_s, and its natural-log normaliser is (M + log2 sum) ln 2.
//
// One thread per (row, head, 8 output elements).  The partial states are in
// entry order, [entry][head of group][D], so for one slot the threads of a
// (row, group) read one contiguous run of G*D elements with 16-byte loads.
// Slots are merged in batches with a running maximum (the same exact merge,
// rescaled whenever the maximum grows), so that each thread issues the loads
// of a whole batch before it uses any of them: the kernel is bound by HBM and
// needs many bytes in flight per SM.
#include "common.cuh"
#include "internal.h"

namespace msa {

template <typename PT>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  uint4 u;
  __device__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ void to_f32(float (&f)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(h[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float (&f)[8]) {
    uint4 u;
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec8<float> {
  float4 a, b;
  __device__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ void to_f32(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  __device__ static void store(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

// Slots merged per batch: their loads are all issued before any is used, so a
// thread keeps kBatch 16-byte partial loads in flight.
constexpr int kBatch = 8;

template <typename PT, typename OT, int D>
__global__ void __launch_bounds__(256) combine_kernel(Problem P, const int32_t* __restrict__ pos,
                                                      const PT* __restrict__ part_o,
                                                      const float* __restrict__ part_lse,
                                                      OT* __restrict__ out,
                                                      float* __restrict__ lse_out) {
  constexpr int CH = D / 8;  // 8-element chunks per head row
  const long long n = (long long)P.T * P.Hq * CH;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int ch = int(idx % CH);
    const long long rh = idx / CH;          // r * Hq + h
    const int h = int(rh % P.Hq);
    const int r = int(rh / P.Hq);
    const int g = h / P.G, hh = h % P.G;
    const int32_t* ps = pos + ((long long)g * P.T + r) * P.K;
    // running merge: M = max lse so far, acc and sum scaled by 2^-M
    float M = -INFINITY, sum = 0.f;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int s0 = 0; s0 < P.K; s0 += kBatch) {
      int e[kBatch];
      float l[kBatch];
      Vec8<PT> v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) e[u] = s0 + u < P.K ? __ldg(ps + s0 + u) : -1;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (e[u] >= 0) {
          const long long prow = (long long)e[u] * P.G + hh;
          l[u] = __ldg(part_lse + prow);
          v[u].load(part_o + prow * D + ch * 8);
        } else {
          l[u] = -INFINITY;
        }
      }
      float bm = l[0];
#pragma unroll
      for (int u = 1; u < kBatch; ++u) bm = fmaxf(bm, l[u]);
      if (bm == -INFINITY) continue;  // no valid slot in this batch
      if (bm > M) {
        const float sc = exp2f(M - bm);  // 0 while M is -inf
        sum *= sc;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= sc;
        M = bm;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (e[u] >= 0) {
          const float w = exp2f(l[u] - M);
          sum += w;
          float f[8];
          v[u].to_f32(f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, f[i], acc[i]);
        }
      }
    }
    if (M != -INFINITY) {
      const float inv = 1.f / sum;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    Vec8<OT>::store(out + rh * D + ch * 8, acc);
    if (lse_out && ch == 0)
      lse_out[rh] = M == -INFINITY ? -INFINITY : (M + log2f(sum)) * 0.6931471805599453f;
  }
}

template <typename T, int D>
static cudaError_t launch_t(const Problem& P, const int32_t* pos, const Partials& part,
                            void* out, float* lse, cudaStream_t s) {
  const long long n = (long long)P.T * P.Hq * (D / 8);
  long long blocks = (n + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
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
