// Merge of the per-slot partial softmax states of one (query row, head).
//
// The KV-outer kernels finish the softmax of each (row, head, slot) over one
// block and store o_s (normalised) and lse_s = log2 of its normaliser, at the
// entry position the block -> query lists gave that (group, row, slot).  The
// exact softmax over the union of the slots' tokens is
//     O = sum_s w_s o_s,   w_s = 2^(lse_s - M) / sum_u 2^(lse_u - M),
// with M = max_s lse_s, and its natural-log normaliser is (M + log2 sum) ln 2.
//
// Two kernels.  For bf16 partial states with 16 heads of 128 dims per slot (a
// slot of one (row, group) is then one contiguous 4 KB run), a loader warp
// brings each slot in with a TMA bulk copy and eight warps merge from shared
// memory: HBM serves these 4 KB runs at scattered positions faster through
// bulk copies than through 16-byte loads.  Otherwise (fp32, other shapes):
// one thread per (row, head, 8 output elements).  The partial states are in
// entry order, [entry][head of group][D], so for one slot the threads of a
// (row, group) read one contiguous run of G*D elements with 16-byte loads.
// Slots are merged in batches with a running maximum (the same exact merge,
// rescaled whenever the maximum grows), so that each thread issues the loads
// of a whole batch before it uses any of them: the kernel is bound by HBM and
// needs many bytes in flight per SM.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

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

// ---------------------------------------------------------------------------
// TMA-fed combine for bf16 partial states with 16 heads of 128 dims per slot
// (one slot of one (row, group) = 16 x 128 bf16 = 4 KB, contiguous).  A loader
// warp brings the slots of a (row, group) into shared memory with one 4 KB
// bulk copy per slot (plus its 64-byte row of log-normalisers), eight slots per
// stage; eight compute warps merge them (thread = head x 16-byte chunk) with a
// running maximum and write the output row.
// ---------------------------------------------------------------------------
namespace {
constexpr int kCBatch = 8;                       // slots per stage
constexpr int kCStages = 3;
constexpr int kCSlotBytes = 16 * 128 * 2;        // 4 KB
constexpr int kCLseBytes = 16 * 4;               // 64 B
constexpr int kCStageBytes = kCBatch * (kCSlotBytes + kCLseBytes);
constexpr int kCThreads = 288;                   // 8 compute warps + 1 loader warp

struct CBars {
  uint64_t full[kCStages], empty[kCStages];
  uint32_t mask[kCStages];                       // valid slots of the stage's batch
  int abort;
};
constexpr size_t kCSmem = 128 + kCStages * kCStageBytes + sizeof(CBars) + 64;
}  // namespace

__global__ void __launch_bounds__(kCThreads, 2)
combine_tma_kernel(Problem P, const int32_t* __restrict__ pos,
                   const __nv_bfloat16* __restrict__ part_o, const float* __restrict__ part_lse,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
                   int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  CBars* bars = reinterpret_cast<CBars*>(smem + kCStages * kCStageBytes);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kCStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 8);
    }
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  const long long units = (long long)P.Hkv * P.T;
  const int nb = (P.K + kCBatch - 1) / kCBatch;     // batches per unit
  bool failed = false;
  if (warp == 8) {
    // ---------------- loader ----------------
    int k = 0;
    tc::ArmedRing armed;  // lane 0: stages it has armed for copies
    for (long long u = blockIdx.x; u < units && !failed; u += gridDim.x) {
      const int32_t* ps = pos + u * P.K;              // pos[g][r][:] with u = g * T + r
      for (int b = 0; b < nb; ++b, ++k) {
        const int st = k % kCStages;
        const int slot = b * kCBatch + lane;
        const int e = (lane < kCBatch && slot < P.K) ? __ldg(ps + slot) : -1;
        const unsigned m = __ballot_sync(MSA_FULL_MASK, e >= 0);
        bool ok = true;
        if (lane == 0) ok = tc::mbar_wait(&bars->empty[st], ((k / kCStages) & 1) ^ 1, abort);
        if (!__shfl_sync(MSA_FULL_MASK, ok, 0)) { failed = true; break; }
        uint8_t* sb = smem + st * kCStageBytes;
        if (lane == 0) {
          bars->mask[st] = m;
          tc::mbar_arrive_expect_tx(&bars->full[st], __popc(m) * (kCSlotBytes + kCLseBytes));
          armed.note(st, (k / kCStages) & 1);
        }
        __syncwarp();
        if (e >= 0) {
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
              ::"r"(tc::smem_addr(sb + lane * kCSlotBytes)),
              "l"(part_o + (long long)e * (kCSlotBytes / 2)), "r"(kCSlotBytes),
              "r"(tc::smem_addr(&bars->full[st]))
              : "memory");
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
              ::"r"(tc::smem_addr(sb + kCBatch * kCSlotBytes + lane * kCLseBytes)),
              "l"(part_lse + (long long)e * 16), "r"(kCLseBytes),
              "r"(tc::smem_addr(&bars->full[st]))
              : "memory");
        }
      }
    }
    // every copy issued has landed before the CTA can leave
    if (lane == 0 && !armed.drain(bars->full)) failed = true;
    if (lane != 0) failed = false;
  } else {
    // ---------------- merge: thread = (head hh, 16-byte chunk ch) ----------------
    const int hh = threadIdx.x >> 4, ch = threadIdx.x & 15;
    int k = 0;
    for (long long u = blockIdx.x; u < units && !failed; u += gridDim.x) {
      float M = -INFINITY, sum = 0.f, acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int b = 0; b < nb; ++b, ++k) {
        const int st = k % kCStages;
        if (!__all_sync(MSA_FULL_MASK,
                        tc::mbar_wait(&bars->full[st], (k / kCStages) & 1, abort))) {
          failed = true;
          break;
        }
        const uint8_t* sb = smem + st * kCStageBytes;
        const unsigned m = bars->mask[st];
        float l[kCBatch];
        uint4 v[kCBatch];
#pragma unroll
        for (int j = 0; j < kCBatch; ++j) {
          if ((m >> j) & 1u) {
            l[j] = reinterpret_cast<const float*>(sb + kCBatch * kCSlotBytes + j * kCLseBytes)[hh];
            v[j] = *reinterpret_cast<const uint4*>(sb + j * kCSlotBytes + hh * 256 + ch * 16);
          } else {
            l[j] = -INFINITY;
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->empty[st]);  // the stage's data is in registers
        float bm = l[0];
#pragma unroll
        for (int j = 1; j < kCBatch; ++j) bm = fmaxf(bm, l[j]);
        if (bm == -INFINITY) continue;
        if (bm > M) {
          const float sc = exp2f(M - bm);  // 0 while M is -inf
          sum *= sc;
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] *= sc;
          M = bm;
        }
#pragma unroll
        for (int j = 0; j < kCBatch; ++j) {
          if ((m >> j) & 1u) {
            const float w = exp2f(l[j] - M);
            sum += w;
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 x = __bfloat1622float2(h2[i]);
              acc[2 * i] = fmaf(w, x.x, acc[2 * i]);
              acc[2 * i + 1] = fmaf(w, x.y, acc[2 * i + 1]);
            }
          }
        }
      }
      if (failed) break;
      if (M != -INFINITY) {
        const float inv = 1.f / sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= inv;
      }
      const int g = int(u / P.T), r = int(u % P.T);
      const long long rh = (long long)r * P.Hq + g * 16 + hh;
      Vec8<__nv_bfloat16>::store(out + rh * 128 + ch * 8, acc);
      if (lse_out && ch == 0)
        lse_out[rh] = M == -INFINITY ? -INFINITY : (M + log2f(sum)) * 0.6931471805599453f;
    }
  }
  if (failed) {
    bars->abort = 1;
    atomicOr(status, tc::kStatusWaitTimeout);
  }
}

static bool combine_tma_supported(const Problem& P) {
  return !P.f32 && P.D == 128 && P.G == 16;
}

static int combine_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
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
                           void* out, float* lse, int32_t* status, cudaStream_t s) {
  if ((long long)P.T * P.Hq == 0) return cudaSuccess;
  if (combine_tma_supported(P)) {
    cudaError_t e = cudaFuncSetAttribute(combine_tma_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(kCSmem));
    if (e != cudaSuccess) return e;
    const long long units = (long long)P.Hkv * P.T;
    const int grid = int(std::min<long long>(2LL * combine_sms(), units));
    combine_tma_kernel<<<grid, kCThreads, kCSmem, s>>>(
        P, pos, static_cast<const __nv_bfloat16*>(part.o), part.lse2,
        static_cast<__nv_bfloat16*>(out), lse, status);
    return cudaGetLastError();
  }
  if (P.f32) return P.D == 64 ? launch_t<float, 64>(P, pos, part, out, lse, s)
                              : launch_t<float, 128>(P, pos, part, out, lse, s);
  return P.D == 64 ? launch_t<__nv_bfloat16, 64>(P, pos, part, out, lse, s)
                   : launch_t<__nv_bfloat16, 128>(P, pos, part, out, lse, s);
}

}  // namespace msa
