// KL-alignment loss of the index branch and its gradients (training side).
//
// snilld.dk "Træning og stabilisering": Top-k is not differentiable, so an
// extra KL-alignment loss trains the index projections; the index branch is
// to match the main branch, whose group-averaged distribution over the selected
// tokens is the teacher, and a gradient detach keeps the loss out of the rest
// of the layer (aiforradalom.online "A betanítás és a kernel-optimalizáció":
// a KL-divergence loss aligns the two distributions).  Per (query row r,
// group g), over the causally visible tokens J of the blocks q2k[g, r, :]:
//   index   p_I = softmax_j(q_idx[r,g] . k_idx[j])                (raw scores)
//   teacher p_T = mean over the group's heads h of softmax_j(scale * q[r,h] . k[j,g])
//   kl      = sum_j p_T[j] (ln p_T[j] - ln p_I[j])
// The loss is the mean of kl over the N = T * Hkv pairs.  With q, k and q2k held
// constant, d loss / d s_j = (p_I[j] - p_T[j]) / N, so dq_idx[r,g] = sum_j ds_j
// k_idx[j] and dk_idx[j] = sum over the pairs holding token j of ds_j q_idx[r,g].
//
//   kl_rows_kernel  one CTA per (row, group), CUDA cores: the teacher's per-head
//                   normalisers (pass 1), the teacher probabilities and index
//                   scores (pass 2), kl, the score gradients ds (kept per (group,
//                   row, slot, offset)) and dq_idx;
//   kl_dk_kernel    KV-outer over the block -> query lists: a block's 128 index
//                   keys collect ds * q_idx over the list's entries and add them
//                   into dk_idx with fp32 atomics (groups and query chunks share
//                   a block's keys);
//   kl_sum_kernel   the mean, summed in a fixed order in fp64.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace msa {

constexpr int kKlThreads = 128;
constexpr int kHB = 8;        // query heads whose logits one pass keeps in registers
constexpr int kDkChunk = 32;  // index dims per accumulation pass of kl_dk_kernel

// Block-wide reductions over kKlThreads threads (scratch: 4 floats).
__device__ __forceinline__ float block_max(float v, float* scratch) {
  v = warp_max_f32(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  return fmaxf(fmaxf(scratch[0], scratch[1]), fmaxf(scratch[2], scratch[3]));
}
__device__ __forceinline__ float block_sum(float v, float* scratch) {
  v = warp_sum_f32(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  return (scratch[0] + scratch[1]) + (scratch[2] + scratch[3]);
}

// scale * q_h . k_row for heads hb .. hb + nh - 1 (q rows in shared memory).
template <typename TQ>
__device__ __forceinline__ void head_logits(const float* __restrict__ qh, int D, int hb, int nh,
                                            const TQ* __restrict__ krow, float scale,
                                            float (&z)[kHB]) {
#pragma unroll
  for (int i = 0; i < kHB; ++i) z[i] = 0.f;
  for (int d0 = 0; d0 < D; d0 += 8) {
    float kv[8];
    load_vec<TQ, 8>(krow + d0, kv);
#pragma unroll
    for (int i = 0; i < kHB; ++i) {
      if (i < nh) {
        const float* qr = qh + (hb + i) * D + d0;
#pragma unroll
        for (int e = 0; e < 8; ++e) z[i] = fmaf(qr[e], kv[e], z[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kHB; ++i) z[i] *= scale;
}

template <typename TQ, typename TI>
__global__ void __launch_bounds__(kKlThreads) kl_rows_kernel(
    Problem P, const TQ* __restrict__ q, const TQ* __restrict__ k, const TI* __restrict__ q_idx,
    const TI* __restrict__ k_idx, const int32_t* __restrict__ q2k, float* __restrict__ kl_rows,
    float* __restrict__ dq_idx, float* __restrict__ ds_buf, int32_t* __restrict__ status) {
  extern __shared__ float smf[];
  const int G = P.G, D = P.D, DI = P.DI, Bk = P.Bk, K = P.K;
  const int n = K * Bk;  // token slots (slot * Bk + offset)
  float* qh = smf;               // [G][D] the group's query heads
  float* qi = qh + G * D;        // [DI]  the index query
  float* hm = qi + DI;           // [G]   teacher max per head
  float* hl = hm + G;            // [G]   teacher normaliser per head
  float* pt = hl + G;            // [n]   teacher probability per token
  float* sc = pt + n;            // [n]   index score, then its gradient ds
  float* red = sc + n;           // [4]   reduction scratch
  __shared__ int blk[32];        // block of each slot, -1 if none

  const int g = int(blockIdx.x / P.T), r = int(blockIdx.x % P.T);
  const int b = r / P.Sq;
  const long long t = P.q_pos0 + r % P.Sq;
  const int tid = threadIdx.x;
  if (tid < K) {
    const int c = q2k[((long long)g * P.T + r) * K + tid];
    const bool ok = c >= 0 && (long long)c <= t / Bk;
    if (!ok && c != -1) atomicOr(status, kStatusBadEntry);
    blk[tid] = ok ? c : -1;
  }
  for (int x = tid; x < G * D; x += kKlThreads)
    qh[x] = to_f32(q[((long long)r * P.Hq + (long long)g * G + x / D) * D + x % D]);
  for (int x = tid; x < DI; x += kKlThreads)
    qi[x] = to_f32(q_idx[((long long)r * P.Hkv + g) * DI + x]);
  __syncthreads();

  // token m of the row: its key index j, or -1 when the slot is empty or j > t
  auto token = [&](int m) -> long long {
    const int c = blk[m / Bk];
    if (c < 0) return -1;
    const long long j = (long long)c * Bk + m % Bk;
    return j <= t ? j : -1;
  };

  // pass 1: per head, the maximum and the normaliser of the scaled logits
  for (int hb = 0; hb < G; hb += kHB) {
    const int nh = min(kHB, G - hb);
    float mx[kHB], sm[kHB];
#pragma unroll
    for (int i = 0; i < kHB; ++i) { mx[i] = -INFINITY; sm[i] = 0.f; }
    for (int m = tid; m < n; m += kKlThreads) {
      const long long j = token(m);
      if (j < 0) continue;
      float z[kHB];
      head_logits<TQ>(qh, D, hb, nh, k + (key_row(P, b, j) * P.Hkv + g) * D, P.scale, z);
#pragma unroll
      for (int i = 0; i < kHB; ++i) {
        if (z[i] > mx[i]) { sm[i] = sm[i] * __expf(mx[i] - z[i]) + 1.f; mx[i] = z[i]; }
        else sm[i] += __expf(z[i] - mx[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kHB; ++i) {
      if (i < nh) {  // uniform over the CTA
        const float M = block_max(mx[i], red);
        const float L = block_sum(mx[i] == -INFINITY ? 0.f : sm[i] * __expf(mx[i] - M), red);
        if (tid == 0) { hm[hb + i] = M; hl[hb + i] = L; }
      }
    }
  }
  __syncthreads();

  // pass 2: teacher probabilities and index scores
  float smax = -INFINITY;
  for (int m = tid; m < n; m += kKlThreads) {
    const long long j = token(m);
    if (j < 0) { pt[m] = 0.f; sc[m] = -INFINITY; continue; }
    float p = 0.f;
    const long long row = key_row(P, b, j);
    const TQ* krow = k + (row * P.Hkv + g) * D;
    for (int hb = 0; hb < G; hb += kHB) {
      const int nh = min(kHB, G - hb);
      float z[kHB];
      head_logits<TQ>(qh, D, hb, nh, krow, P.scale, z);
#pragma unroll
      for (int i = 0; i < kHB; ++i)
        if (i < nh) p += __expf(z[i] - hm[hb + i]) / hl[hb + i];
    }
    pt[m] = p / G;
    const TI* irow = k_idx + row * DI;
    float s = 0.f;
    for (int d0 = 0; d0 < DI; d0 += 8) {
      float kv[8];
      load_vec<TI, 8>(irow + d0, kv);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(qi[d0 + e], kv[e], s);
    }
    sc[m] = s;
    smax = fmaxf(smax, s);
  }
  const float S = block_max(smax, red);
  float se = 0.f;
  for (int m = tid; m < n; m += kKlThreads)
    if (sc[m] != -INFINITY) se += __expf(sc[m] - S);
  const float lse = S + __logf(block_sum(se, red));

  // pass 3: kl and ds = (p_I - p_T) / N, kept per (group, row, slot, offset)
  const float inv_n = 1.f / (float(P.T) * float(P.Hkv));
  float klp = 0.f;
  float* dsrow = ds_buf + ((long long)g * P.T + r) * n;
  for (int m = tid; m < n; m += kKlThreads) {
    float ds = 0.f;
    if (sc[m] != -INFINITY) {
      const float lpi = sc[m] - lse;
      if (pt[m] > 0.f) klp += pt[m] * (__logf(pt[m]) - lpi);
      ds = (__expf(lpi) - pt[m]) * inv_n;
    }
    if (blk[m / Bk] >= 0) dsrow[m] = ds;
    sc[m] = ds;
  }
  const float kl = block_sum(klp, red);
  if (tid == 0) kl_rows[(long long)g * P.T + r] = kl;
  __syncthreads();

  // dq_idx[r, g, d] = sum_j ds_j k_idx[j, d]: thread d walks the tokens
  for (int d = tid; d < DI; d += kKlThreads) {
    float acc = 0.f;
    for (int m = 0; m < n; ++m) {
      const long long j = token(m);
      if (j >= 0) acc = fmaf(sc[m], to_f32(k_idx[key_row(P, b, j) * DI + d]), acc);
    }
    dq_idx[((long long)r * P.Hkv + g) * DI + d] = acc;
  }
}

// dk_idx over the block -> query lists: thread = key offset inside the block.
template <typename TI>
__global__ void __launch_bounds__(kKlThreads) kl_dk_kernel(Problem P, const TI* __restrict__ q_idx,
                                                           const float* __restrict__ ds_buf,
                                                           Lists L, float* __restrict__ dk_idx) {
  __shared__ float qs[32][kDkChunk];
  __shared__ int rows_s[32], slots_s[32];
  const int DI = P.DI, off = threadIdx.x;
  for (long long lid = blockIdx.x; lid < P.nlists; lid += gridDim.x) {
    const int e0 = L.list_off[lid], e1 = L.list_off[lid + 1];
    if (e0 == e1) continue;
    const int c = int(lid % P.nblk);
    const long long rest = lid / P.nblk;  // (b * Hkv + g) * nqc + qc
    const int g = int((rest / P.nqc) % P.Hkv);
    const int b = int(rest / ((long long)P.nqc * P.Hkv));
    const long long j = (long long)c * P.Bk + off;
    for (int d0 = 0; d0 < DI; d0 += kDkChunk) {
      float acc[kDkChunk];
#pragma unroll
      for (int i = 0; i < kDkChunk; ++i) acc[i] = 0.f;
      for (int eb = e0; eb < e1; eb += 32) {
        const int ne = min(32, e1 - eb);
        __syncthreads();  // the previous batch is consumed
        if (threadIdx.x < ne) {
          const int packed = L.entries[eb + threadIdx.x];
          rows_s[threadIdx.x] = packed >> 5;
          slots_s[threadIdx.x] = packed & 31;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < ne * kDkChunk; x += kKlThreads) {
          const int e = x / kDkChunk, d = d0 + x % kDkChunk;  // DI is a multiple of 32
          qs[e][x % kDkChunk] = to_f32(q_idx[((long long)rows_s[e] * P.Hkv + g) * DI + d]);
        }
        __syncthreads();
        for (int e = 0; e < ne; ++e) {
          const float ds =
              ds_buf[(((long long)g * P.T + rows_s[e]) * P.K + slots_s[e]) * P.Bk + off];
#pragma unroll
          for (int i = 0; i < kDkChunk; ++i) acc[i] = fmaf(ds, qs[e][i], acc[i]);
        }
      }
      if (j < P.Skv) {
        float* dst = dk_idx + (block_row(P, b, c) + off) * DI + d0;
#pragma unroll
        for (int i = 0; i < kDkChunk; ++i) atomicAdd(dst + i, acc[i]);
      }
    }
  }
}

// loss = (sum of kl_rows) / N, summed in a fixed order in fp64.
__global__ void __launch_bounds__(1024) kl_sum_kernel(const float* __restrict__ kl_rows,
                                                      long long n, float* __restrict__ loss) {
  __shared__ double part[32];
  double acc = 0.0;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) acc += double(kl_rows[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(MSA_FULL_MASK, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) s += part[w];
    *loss = float(s / double(n));
  }
}

size_t kl_rows_smem(const Problem& P) {
  return sizeof(float) * (size_t(P.G) * P.D + P.DI + 2 * P.G + 2 * size_t(P.K) * P.Bk + 4);
}

template <typename TQ, typename TI>
static cudaError_t launch_kl_t(const Problem& P, const void* q, const void* k, const void* q_idx,
                               const void* k_idx, const int32_t* q2k, const Lists& L,
                               float* kl_rows, float* ds_buf, float* loss, float* dq_idx,
                               float* dk_idx, int32_t* status, cudaStream_t s) {
  const size_t smem = kl_rows_smem(P);
  auto rows = kl_rows_kernel<TQ, TI>;
  cudaError_t e =
      cudaFuncSetAttribute(rows, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned pairs = unsigned((long long)P.T * P.Hkv);
  rows<<<pairs, kKlThreads, smem, s>>>(P, (const TQ*)q, (const TQ*)k, (const TI*)q_idx,
                                       (const TI*)k_idx, q2k, kl_rows, dq_idx, ds_buf, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = cudaMemsetAsync(dk_idx, 0, sizeof(float) * size_t(P.kv_rows) * P.DI, s);
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(std::min<long long>(P.nlists, 148LL * 16));
  kl_dk_kernel<TI><<<grid, kKlThreads, 0, s>>>(P, (const TI*)q_idx, ds_buf, L, dk_idx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kl_sum_kernel<<<1, 1024, 0, s>>>(kl_rows, pairs, loss);
  return cudaGetLastError();
}

bool index_kl_supported(const Problem& P) {
  return !P.idx4 && kl_rows_smem(P) <= 200 * 1024 && P.D % 8 == 0 && P.DI % kDkChunk == 0 &&
         P.Bk == kKlThreads && P.K <= 32;
}

cudaError_t launch_index_kl(const Problem& P, const void* q, const void* k, const void* q_idx,
                            const void* k_idx, const int32_t* q2k, const Lists& L,
                            float* kl_rows, float* ds_buf, float* loss, float* dq_idx,
                            float* dk_idx, int32_t* status, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  using fp8 = __nv_fp8_e4m3;
  if (P.f32)
    return launch_kl_t<float, float>(P, q, k, q_idx, k_idx, q2k, L, kl_rows, ds_buf, loss,
                                     dq_idx, dk_idx, status, s);
  if (P.qk8)
    return P.idx8 ? launch_kl_t<fp8, fp8>(P, q, k, q_idx, k_idx, q2k, L, kl_rows, ds_buf, loss,
                                          dq_idx, dk_idx, status, s)
                  : launch_kl_t<fp8, bf16>(P, q, k, q_idx, k_idx, q2k, L, kl_rows, ds_buf, loss,
                                           dq_idx, dk_idx, status, s);
  return P.idx8 ? launch_kl_t<bf16, fp8>(P, q, k, q_idx, k_idx, q2k, L, kl_rows, ds_buf, loss,
                                         dq_idx, dk_idx, status, s)
                : launch_kl_t<bf16, bf16>(P, q, k, q_idx, k_idx, q2k, L, kl_rows, ds_buf, loss,
                                          dq_idx, dk_idx, status, s);
}

}  // namespace msa
