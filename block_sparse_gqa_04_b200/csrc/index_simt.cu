// Index branch on CUDA cores: raw index scores q_idx . k_idx over the visible
// tokens of each 128-token block, max-pooled per block without ever storing a
// token score ("Substantial numerical differences with Minimax MSA attention vs
// Minimax's Reference", section 原因分析: amax over the block axis, kept per
// index head; snilld.dk "Hvad er MSA i praksis": one index-query head per GQA
// group against one shared index-key head).
//
// Two shapes of work:
//  * index_rows_kernel: one thread per query row, a CTA per (128-row tile,
//    block).  Used for fp32 problems and index dims the tensor-core kernel does
//    not cover.
//  * index_keys_kernel: one thread per key token, a CTA per (sequence, block),
//    for a handful of query rows per sequence (decode).  This streams k_idx once
//    at HBM speed, which is what bounds decode.
#include "common.cuh"
#include "internal.h"

namespace msa {

__global__ void fill_kernel(float* __restrict__ p, size_t n, float value) {
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x)
    p[i] = value;
}

cudaError_t launch_fill(float* p, size_t n, float value, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  fill_kernel<<<unsigned(blocks), 256, 0, s>>>(p, n, value);
  return cudaGetLastError();
}

// grid (nblk, ceil(Sq/128), B), 128 threads; dynamic smem 128*DI floats.
template <typename T, int DI>
__global__ void __launch_bounds__(128) index_rows_kernel(Problem P, const T* __restrict__ q_idx,
                                                         const T* __restrict__ k_idx,
                                                         float* __restrict__ bmax) {
  extern __shared__ float ks[];  // [Bk][DI]
  const int c = blockIdx.x;
  const int tile = blockIdx.y;
  const int b = blockIdx.z;
  const int i = tile * 128 + threadIdx.x;
  const int i_last = min(P.Sq - 1, tile * 128 + 127);
  const long long t_last = P.q_pos0 + i_last;
  const long long j0 = (long long)c * P.Bk;
  if (j0 > t_last) return;  // no row of this tile sees block c
  const int nkeys = (int)min((long long)P.Bk, (long long)P.Skv - j0);
  const T* kb = k_idx + block_row(P, b, c) * DI;
  for (int e = threadIdx.x; e < nkeys * DI; e += blockDim.x) ks[e] = to_f32(kb[e]);
  __syncthreads();
  if (i >= P.Sq) return;
  const long long t = P.q_pos0 + i;
  const int r = b * P.Sq + i;
  // visible keys of this block for row t
  const int jn = (int)max(0LL, min((long long)nkeys, t - j0 + 1));
  const T* qrow = q_idx + (long long)r * P.Hkv * DI;
  for (int g = 0; g < P.Hkv; ++g) {
    float qv[DI];
    load_vec<T, DI>(qrow + g * DI, qv);
    float m = -INFINITY;
    for (int j = 0; j < jn; ++j) {
      const float* kr = ks + j * DI;
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DI; ++d) acc = fmaf(qv[d], kr[d], acc);
      m = fmaxf(m, acc);
    }
    bmax[((long long)g * P.T + r) * P.nblk + c] = m;
  }
}

// grid (nblk, B), 128 threads (one key each); smem holds the rows' index
// queries as fp32 [Sq][Hkv][DI].
template <typename T, int DI>
__global__ void __launch_bounds__(128) index_keys_kernel(Problem P, const T* __restrict__ q_idx,
                                                         const T* __restrict__ k_idx,
                                                         float* __restrict__ bmax) {
  extern __shared__ float qs[];
  __shared__ float red[4];
  const int c = blockIdx.x;
  const int b = blockIdx.y;
  const long long j0 = (long long)c * P.Bk;
  const long long t_last = P.q_pos0 + P.Sq - 1;
  if (j0 > t_last) return;
  const int nq = P.Sq * P.Hkv * DI;
  const T* qb = q_idx + (long long)b * nq;
  for (int e = threadIdx.x; e < nq; e += blockDim.x) qs[e] = to_f32(qb[e]);
  const long long j = j0 + threadIdx.x;
  const bool in_seq = threadIdx.x < P.Bk && j < P.Skv;
  float kv[DI];
  if (in_seq) {
    load_vec<T, DI>(k_idx + key_row(P, b, j) * DI, kv);
  } else {
#pragma unroll
    for (int d = 0; d < DI; ++d) kv[d] = 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = 0; i < P.Sq; ++i) {
    const long long t = P.q_pos0 + i;
    const bool vis = in_seq && j <= t;
    for (int g = 0; g < P.Hkv; ++g) {
      const float* qv = qs + (i * P.Hkv + g) * DI;
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DI; ++d) acc = fmaf(kv[d], qv[d], acc);
      float m = warp_max_f32(vis ? acc : -INFINITY);
      if (lane == 0) red[warp] = m;
      __syncthreads();
      if (threadIdx.x == 0) {
        float mm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        if (j0 <= t) bmax[((long long)g * P.T + (long long)b * P.Sq + i) * P.nblk + c] = mm;
      }
      __syncthreads();
    }
  }
}

template <typename T, int DI>
static cudaError_t launch_rows(const Problem& P, const void* q_idx, const void* k_idx,
                               float* bmax, cudaStream_t s) {
  size_t smem = size_t(P.Bk) * DI * sizeof(float);
  auto kern = index_rows_kernel<T, DI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(P.nblk, (P.Sq + 127) / 128, P.B);
  kern<<<grid, 128, smem, s>>>(P, (const T*)q_idx, (const T*)k_idx, bmax);
  return cudaGetLastError();
}

template <typename T, int DI>
static cudaError_t launch_keys(const Problem& P, const void* q_idx, const void* k_idx,
                               float* bmax, cudaStream_t s) {
  size_t smem = size_t(P.Sq) * P.Hkv * DI * sizeof(float);
  auto kern = index_keys_kernel<T, DI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(P.nblk, P.B);
  kern<<<grid, 128, smem, s>>>(P, (const T*)q_idx, (const T*)k_idx, bmax);
  return cudaGetLastError();
}

// Key-parallel when the query rows of a sequence are few enough for their
// index queries to sit in shared memory.
static bool use_keys_kernel(const Problem& P) {
  return P.Sq <= 8 && size_t(P.Sq) * P.Hkv * P.DI * sizeof(float) <= 96 * 1024;
}

template <typename T>
static cudaError_t dispatch_di(const Problem& P, const void* qi, const void* ki, float* bm,
                               cudaStream_t s) {
  const bool keys = use_keys_kernel(P);
  switch (P.DI) {
    case 32: return keys ? launch_keys<T, 32>(P, qi, ki, bm, s) : launch_rows<T, 32>(P, qi, ki, bm, s);
    case 64: return keys ? launch_keys<T, 64>(P, qi, ki, bm, s) : launch_rows<T, 64>(P, qi, ki, bm, s);
    case 128: return keys ? launch_keys<T, 128>(P, qi, ki, bm, s) : launch_rows<T, 128>(P, qi, ki, bm, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_index_simt(const Problem& P, const void* q_idx, const void* k_idx,
                              float* bmax, cudaStream_t s) {
  if (P.idx4) return cudaErrorInvalidValue;  // NVFP4 codes go through nvfp4.cu
  if (P.idx8) return dispatch_di<__nv_fp8_e4m3>(P, q_idx, k_idx, bmax, s);
  return P.f32 ? dispatch_di<float>(P, q_idx, k_idx, bmax, s)
               : dispatch_di<__nv_bfloat16>(P, q_idx, k_idx, bmax, s);
}

}  // namespace msa
