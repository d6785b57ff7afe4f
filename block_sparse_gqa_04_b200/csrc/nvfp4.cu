// NVFP4 index tensors ("MiniMax új eljárása ..." (aiforradalom.online), section
// "Elérhetőség": the MSA kernels come in BF16, FP8, NVFP4 and FP4).  q_idx and
// k_idx hold e2m1 codes, two per byte (element 2i in the low nibble), with one
// unsigned e4m3 scale byte per 16 consecutive elements of index_dim; a value is
// e2m1(code) x ue4m3(scale).
//
// Every such value is exact in bf16 (at most 5 significant bits, exponents
// between 2^-10 and 2^11), so the index branch can take two routes with the same
// result as the bf16 kernels on the decoded values:
//  * dequant_nvfp4_kernel decodes into a bf16 copy in the workspace, which the
//    tensor-core index kernels then read (prefill: the GEMM is bound by the
//    tensor pipe, and the decode pass adds ~0.2 GB of traffic at 128K);
//  * index_keys_nvfp4_kernel decodes each key in registers while streaming
//    k_idx once (decode rows: the step is bound by the k_idx read, which NVFP4
//    makes 3.6x smaller than bf16).
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

// e2m1 code (4 bits: sign, 2 exponent bits with bias 1, 1 mantissa bit) to
// fp32 bits: exponent 0 is subnormal, mantissa x 0.5.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const uint32_t mag = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3f000000u : 0u);
  return __uint_as_float(mag | ((c & 8u) << 28));
}

// ue4m3 scale byte (4 exponent bits with bias 7, 3 mantissa bits, no sign) to
// fp32; exponent 0 is subnormal (mantissa / 8 x 2^-6).
__device__ __forceinline__ float ue4m3_to_f32(uint32_t s) {
  const uint32_t e = (s >> 3) & 15u, m = s & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * 0.001953125f;
}

// Two fp32 values as bf16x2 (a in the low half); the values decoded here are
// exact in bf16, so the rounding (to nearest even) never changes them.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// The 16 values of one group: 8 code bytes and its scale.
__device__ __forceinline__ void decode_group(uint2 codes, uint32_t scale, float (&out)[16]) {
  const float s = ue4m3_to_f32(scale);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t byte = ((i < 4 ? codes.x : codes.y) >> (8 * (i & 3))) & 0xffu;
    out[2 * i] = e2m1_to_f32(byte & 15u) * s;      // exact: e2m1 x ue4m3 fits fp32
    out[2 * i + 1] = e2m1_to_f32(byte >> 4) * s;
  }
}

// One thread per 16-element group: 8 code bytes + 1 scale in, 32 bytes of bf16 out.
__global__ void __launch_bounds__(256) dequant_nvfp4_kernel(const uint2* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales,
                                                            uint4* __restrict__ out,
                                                            long long groups) {
  for (long long gi = blockIdx.x * 256LL + threadIdx.x; gi < groups;
       gi += (long long)gridDim.x * 256) {
    float v[16];
    decode_group(codes[gi], scales[gi], v);
    uint4 a, b;
    a.x = pack_bf16(v[0], v[1]);
    a.y = pack_bf16(v[2], v[3]);
    a.z = pack_bf16(v[4], v[5]);
    a.w = pack_bf16(v[6], v[7]);
    b.x = pack_bf16(v[8], v[9]);
    b.y = pack_bf16(v[10], v[11]);
    b.z = pack_bf16(v[12], v[13]);
    b.w = pack_bf16(v[14], v[15]);
    out[2 * gi] = a;
    out[2 * gi + 1] = b;
  }
}

// Decode rows: a CTA of 128 threads takes kKB consecutive blocks of one
// sequence (seven CTAs per SM), thread t the key at offset t of each of them, and the sequence's
// rg = q_len x num_kv_heads (row, group) pairs (at most kMaxRG).  The decoded
// index queries sit in shared memory as fp32 [rg][DI].  Per 16-element group,
// the thread decodes its keys' e2m1 codes through a 16-entry table in shared
// memory (one load per element, no arithmetic), takes the 16-term dot product
// with each pair's query chunk (one 64-byte chunk read serves all its keys),
// and adds it times the key's group scale.  Then a CTA maximum per (block,
// pair) over the visible keys.
constexpr int kKB = 2;  // 4 halves the occupancy and ran 32 % slower at 128K decode
constexpr int kMaxRG = 8;

template <int DI>
__global__ void __launch_bounds__(128, 7) index_keys_nvfp4_kernel(Problem P,
                                                               const uint8_t* __restrict__ qc,
                                                               const uint8_t* __restrict__ kc,
                                                               float* __restrict__ bmax) {
  constexpr int NG = DI / 16;  // scale groups per row
  extern __shared__ float qs[];  // [rg][DI]
  __shared__ float lut[16];
  __shared__ float red[4][kKB][kMaxRG];
  const int b = blockIdx.y;
  const int c0 = blockIdx.x * kKB;
  const long long t_last = P.q_pos0 + P.Sq - 1;
  if ((long long)c0 * P.Bk > t_last) return;  // no row sees these blocks
  const int rgn = P.Sq * P.Hkv;
  if (threadIdx.x < 16) lut[threadIdx.x] = e2m1_to_f32(threadIdx.x);
  // index queries of sequence b: rgn rows of NG groups, decoded
  const int nqg = rgn * NG;
  const long long qg0 = (long long)b * nqg;
  for (int gi = threadIdx.x; gi < nqg; gi += blockDim.x) {
    float v[16];
    decode_group(reinterpret_cast<const uint2*>(qc)[qg0 + gi], P.qsc[qg0 + gi], v);
#pragma unroll
    for (int x = 0; x < 16; ++x) qs[gi * 16 + x] = v[x];
  }
  const int t = threadIdx.x;
  const uint2* kr[kKB];
  const uint8_t* ks[kKB];
  bool have[kKB];
#pragma unroll
  for (int kb = 0; kb < kKB; ++kb) {
    const int c = c0 + kb;
    const long long j = (long long)c * P.Bk + t;
    have[kb] = t < P.Bk && c < P.nblk && j < P.Skv && j <= t_last;
    const long long row = have[kb] ? key_row(P, b, j) : 0;
    kr[kb] = reinterpret_cast<const uint2*>(kc) + row * NG;
    ks[kb] = P.ksc + row * NG;
  }
  __syncthreads();
  float acc[kKB][kMaxRG];
#pragma unroll
  for (int kb = 0; kb < kKB; ++kb)
#pragma unroll
    for (int r = 0; r < kMaxRG; ++r) acc[kb][r] = 0.f;
  for (int grp = 0; grp < NG; ++grp) {
    float kv[kKB][16];
    float sk[kKB];
#pragma unroll
    for (int kb = 0; kb < kKB; ++kb) {
      const uint2 w = have[kb] ? kr[kb][grp] : make_uint2(0u, 0u);
      sk[kb] = have[kb] ? ue4m3_to_f32(ks[kb][grp]) : 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t byte = ((i < 4 ? w.x : w.y) >> (8 * (i & 3))) & 0xffu;
        kv[kb][2 * i] = lut[byte & 15u];
        kv[kb][2 * i + 1] = lut[byte >> 4];
      }
    }
#pragma unroll
    for (int r = 0; r < kMaxRG; ++r) {
      if (r < rgn) {
        const float4* qp = reinterpret_cast<const float4*>(qs + r * DI + grp * 16);
        float q[16];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 f = qp[x];
          q[4 * x] = f.x;
          q[4 * x + 1] = f.y;
          q[4 * x + 2] = f.z;
          q[4 * x + 3] = f.w;
        }
#pragma unroll
        for (int kb = 0; kb < kKB; ++kb) {
          float part = 0.f;
#pragma unroll
          for (int x = 0; x < 16; ++x) part = fmaf(kv[kb][x], q[x], part);
          acc[kb][r] = fmaf(part, sk[kb], acc[kb][r]);
        }
      }
    }
  }
  // maximum over the visible keys of each (block, pair): warps, then the CTA
  const int warp = t >> 5, lane = t & 31;
#pragma unroll
  for (int kb = 0; kb < kKB; ++kb) {
    const long long j = (long long)(c0 + kb) * P.Bk + t;
#pragma unroll
    for (int r = 0; r < kMaxRG; ++r) {
      if (r < rgn) {
        const long long tr = P.q_pos0 + r / P.Hkv;
        const float m = warp_max_f32(have[kb] && j <= tr ? acc[kb][r] : -INFINITY);
        if (lane == 0) red[warp][kb][r] = m;
      }
    }
  }
  __syncthreads();
  if (t < kKB * rgn) {
    const int kb = t / rgn, r = t % rgn;
    const int c = c0 + kb;
    const int i = r / P.Hkv, g = r % P.Hkv;
    if (c < P.nblk && (long long)c * P.Bk <= P.q_pos0 + i) {
      const float mm = fmaxf(fmaxf(red[0][kb][r], red[1][kb][r]), fmaxf(red[2][kb][r], red[3][kb][r]));
      bmax[((long long)g * P.T + (long long)b * P.Sq + i) * P.nblk + c] = mm;
    }
  }
}

template <int DI>
cudaError_t launch_keys(const Problem& P, const void* qc, const void* kc, float* bmax,
                        cudaStream_t s) {
  const size_t smem = size_t(P.Sq) * P.Hkv * DI * sizeof(float);
  auto kern = index_keys_nvfp4_kernel<DI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((P.nblk + kKB - 1) / kKB, P.B);
  kern<<<grid, 128, smem, s>>>(P, static_cast<const uint8_t*>(qc),
                               static_cast<const uint8_t*>(kc), bmax);
  return cudaGetLastError();
}

}  // namespace

bool nvfp4_keys_supported(const Problem& P) {
  return P.idx4 && P.Bk <= 128 && P.Sq * P.Hkv <= kMaxRG;
}

cudaError_t launch_index_nvfp4_keys(const Problem& P, const void* q_codes, const void* k_codes,
                                    float* bmax, cudaStream_t s) {
  if (P.T == 0) return cudaSuccess;
  switch (P.DI) {
    case 32: return launch_keys<32>(P, q_codes, k_codes, bmax, s);
    case 64: return launch_keys<64>(P, q_codes, k_codes, bmax, s);
    case 128: return launch_keys<128>(P, q_codes, k_codes, bmax, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_dequant_nvfp4(const void* codes, const uint8_t* scales, void* out_bf16,
                                 long long rows, int di, cudaStream_t s) {
  const long long groups = rows * (di / 16);
  if (groups == 0) return cudaSuccess;
  long long blocks = (groups + 255) / 256;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  dequant_nvfp4_kernel<<<unsigned(blocks), 256, 0, s>>>(static_cast<const uint2*>(codes), scales,
                                                         static_cast<uint4*>(out_bf16), groups);
  return cudaGetLastError();
}

}  // namespace msa
