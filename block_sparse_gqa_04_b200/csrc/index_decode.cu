// Index branch for a few query rows per sequence (decode): block maxima of the
// raw index scores q_idx . k_idx over the visible tokens of every 128-token
// block ("Substantial numerical differences with Minimax MSA attention vs
// Minimax's Reference", section 原因分析: amax over each block, per index
// head; snilld.dk "Hvad er MSA i praksis": one index-query head per GQA group,
// one shared index-key head).
//
// With one query per sequence the work is a stream over k_idx (0.25 KB per key)
// with a handful of dot products per key, so it is bound by HBM.  The dot
// products run on the tensor cores so that no SM spends more than a few
// cycles per key: for each (sequence, block) item one tcgen05 MMA computes
//     D[128 keys x N] = k_idx_block[128 keys x 128 dims] . Q[N x 128 dims]^T
// with the block's keys on the TMEM lanes and the sequence's RG = rows x groups
// index queries (zero-padded to N columns) on the TMEM columns.
//   * warp 0 streams the k_idx block by TMA (128-byte swizzle) into a ring of
//     shared-memory stages and writes the sequence's queries next to it in the
//     same swizzled K-major layout (they stay in registers while the sequence
//     does not change);
//   * warp 1 issues the MMAs (A = keys, B = queries, both K-major) into one of
//     four N-column TMEM accumulators;
//   * warps 2-5 (one TMEM lane quarter each) read their keys' N scores, mask
//     the keys a row cannot see, reduce each column with a warp redux over
//     orderable keys and combine the four warps' maxima through shared memory.
// Persistent CTAs (two per SM for the bf16 16-wide form, three for fp8, whose
// stages are half the size) take contiguous ranges of items, so consecutive
// items mostly share one sequence.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kKHalf = 128 * 128;      // 128-byte rows x 128 keys (one swizzle span)
constexpr int kThreads = 192;
constexpr int kSlots = 4;               // TMEM accumulators
constexpr int kMaxRG = 32;              // (rows per sequence) x groups handled

// N: padded query width (16 or 32); FP8: fp8 e4m3 index tensors (one 128-byte
// half per row, kind::f8f6f4) instead of bf16 (two halves, kind::f16).
template <int N, bool FP8>
struct Cfg {
  static constexpr int kHalves = FP8 ? 1 : 2;            // 128-byte halves of a row
  static constexpr int kRowChunks = 8 * kHalves;          // 16-byte chunks of a row
  static constexpr int kKBytes = kHalves * kKHalf;        // one block of k_idx
  static constexpr int kSteps = FP8 ? 4 : 8;              // K steps of 32 bytes
  // Several CTAs per SM, each with its own TMA stream (more streams per SM move
  // more bytes): 16-wide bf16 tiles two, fp8 tiles (18-20 KB stages) three;
  // 32-wide bf16 tiles need more shared memory per stage and run one
  static constexpr int kStages = FP8 ? 3 : (N <= 16 ? 3 : 5);
  static constexpr int kCtasPerSm = FP8 ? 3 : (N <= 16 ? 2 : 1);
  static constexpr int kQHalf = N * 128;                  // 128-byte rows of N padded queries
  static constexpr int kStageBytes = kKBytes + kHalves * kQHalf;
  static constexpr uint32_t kTmemCols = kSlots * N < 32 ? 32 : kSlots * N;
  static constexpr uint32_t kIdesc =
      FP8 ? tc::idesc_e4m3_f32(128, N) : tc::idesc_bf16_f32(128, N, 0, 0);
  static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
};

template <int N, bool FP8>
struct Shared {
  uint64_t full[Cfg<N, FP8>::kStages], empty[Cfg<N, FP8>::kStages];
  uint64_t acc_full[kSlots], acc_empty[kSlots];
  uint32_t red[kSlots][4][N];   // per accumulator: the four warps' column maxima
  int qseq[Cfg<N, FP8>::kStages];  // sequence whose queries each stage holds (-1: none)
  uint64_t mma_done;       // the MMA thread's final commit (drain before TMEM is freed)
  uint32_t tmem_base;
  int abort;
};

template <int N, bool FP8>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<N, FP8>::kStages * Cfg<N, FP8>::kStageBytes + sizeof(Shared<N, FP8>) + 64;
}
// two CTAs per SM must fit in the SM's 228 KB where kCtasPerSm is 2
static_assert(smem_bytes<16, false>() <= 116736, "two CTAs per SM");
static_assert(smem_bytes<32, false>() <= 232448, "one CTA per SM");
static_assert(smem_bytes<16, true>() <= 77824, "three CTAs per SM");
static_assert(smem_bytes<32, true>() <= 77824, "three CTAs per SM");

// Barrier of the four epilogue warps that also returns whether any of their
// threads passed `v` (so that they leave together on a failed wait).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

template <int N, bool FP8>
__global__ void __launch_bounds__(kThreads, 2)
index_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, Problem P,
                    const uint8_t* __restrict__ q_idx, float* __restrict__ bmax,
                    int* __restrict__ status, int nvis) {
  using C = Cfg<N, FP8>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  Shared<N, FP8>* sh = reinterpret_cast<Shared<N, FP8>*>(smem + S * C::kStageBytes);
  volatile int* abort = &sh->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int RG = P.Sq * P.Hkv;

  // zero the padded query rows RG..N-1 of every stage once; only rows < RG are
  // rewritten later
  for (int e = threadIdx.x; e < S * C::kHalves * (N - RG) * 8; e += kThreads) {
    const int st = e / (C::kHalves * (N - RG) * 8), rem = e % (C::kHalves * (N - RG) * 8);
    const int h = rem / ((N - RG) * 8), x = rem % ((N - RG) * 8);
    *reinterpret_cast<uint4*>(stages + st * C::kStageBytes + C::kKBytes + h * C::kQHalf +
                              RG * 128 + x * 16) = make_uint4(0, 0, 0, 0);
  }
  tc::fence_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&sh->full[s], 2);   // TMA bytes + the queries written by warp 0
      tc::mbar_init(&sh->empty[s], 1);
      sh->qseq[s] = -1;
    }
    for (int s = 0; s < kSlots; ++s) {
      tc::mbar_init(&sh->acc_full[s], 1);
      tc::mbar_init(&sh->acc_empty[s], 4);
    }
    tc::mbar_init(&sh->mma_done, 1);
    sh->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tc::tma_prefetch(&tmap_k);
  if (warp == 1) tc::tmem_alloc(&sh->tmem_base, C::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  const long long items = (long long)P.B * nvis;
  const long long i0 = items * blockIdx.x / gridDim.x;
  const long long i1 = items * (blockIdx.x + 1) / gridDim.x;
  bool failed = false;

  if (warp == 0) {
    // ---------------- producer: k_idx by TMA, queries from registers ----------------
    constexpr int kQv = N * C::kRowChunks / 32;  // 16-byte query chunks per lane, at most
    uint4 qv[kQv];
    int qb = -1;
    int k = 0;
    tc::ArmedRing armed;  // lane 0: stages whose k_idx copy it issued
    for (long long it = i0; it < i1; ++it, ++k) {
      const int s = k % S;
      const uint32_t ph = (k / S) & 1;
      const int b = int(it / nvis), c = int(it % nvis);
      if (b != qb) {
        const uint4* src =
            reinterpret_cast<const uint4*>(q_idx + (long long)b * RG * C::kRowChunks * 16);
#pragma unroll
        for (int x = 0; x < kQv; ++x) {
          const int e = lane + 32 * x;
          qv[x] = e < RG * C::kRowChunks ? __ldg(src + e) : make_uint4(0, 0, 0, 0);
        }
        qb = b;
      }
      bool ok = true;
      if (lane == 0) ok = tc::mbar_wait(&sh->empty[s], ph ^ 1, abort);
      if (!__shfl_sync(MSA_FULL_MASK, ok, 0)) { failed = true; break; }
      uint8_t* st = stages + s * C::kStageBytes;
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&sh->full[s], C::kKBytes);
        armed.note(s, ph);
        const int row = int(block_row(P, b, c));
        tc::tma_load_2d(st, &tmap_k, &sh->full[s], 0, row);
        if (!FP8) tc::tma_load_2d(st + kKHalf, &tmap_k, &sh->full[s], 64, row);
      }
      // query chunk e = (row n, 16-byte chunk j of its 256 B): K-major, 128-byte
      // swizzle, the layout TMA gives the key block.  A stage that already
      // holds this sequence's queries keeps them.
      const bool put_q = sh->qseq[s] != b;
      if (put_q) {
#pragma unroll
        for (int x = 0; x < kQv; ++x) {
          const int e = lane + 32 * x;
          if (e < RG * C::kRowChunks) {
            const int n = e / C::kRowChunks, j = e % C::kRowChunks;
            *reinterpret_cast<uint4*>(st + C::kKBytes + (j >> 3) * C::kQHalf + n * 128 +
                                      (((j & 7) ^ (n & 7)) << 4)) = qv[x];
          }
        }
        tc::fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        if (put_q) sh->qseq[s] = b;
        tc::mbar_arrive(&sh->full[s]);
      }
    }
    // every copy issued has landed before the CTA can leave (each armed stage
    // also got the second arrival, right after its copy was issued)
    if (lane == 0 && !armed.drain(sh->full)) failed = true;
    if (lane != 0) failed = false;
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int k = 0;
      for (long long it = i0; it < i1; ++it, ++k) {
        const int s = k % S, slot = k % kSlots;
        if (!tc::mbar_wait(&sh->full[s], (k / S) & 1, abort)) { failed = true; break; }
        if (!tc::mbar_wait(&sh->acc_empty[slot], ((k / kSlots) & 1) ^ 1, abort)) {
          failed = true;
          break;
        }
        tc::tc_fence_after();
        const uint32_t kb = tc::smem_addr(stages + s * C::kStageBytes);
        const uint32_t qbase = kb + C::kKBytes;
#pragma unroll
        for (int kk = 0; kk < C::kSteps; ++kk) {
          const uint64_t ad = tc::sdesc_sw128(kb + (kk >> 2) * kKHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t bd =
              tc::sdesc_sw128(qbase + (kk >> 2) * C::kQHalf + (kk & 3) * 32, 16, 1024);
          if (FP8)
            tc::mma_ss_f8(tmem + slot * N, ad, bd, C::kIdesc, kk > 0 ? 1u : 0u);
          else
            tc::mma_ss(tmem + slot * N, ad, bd, C::kIdesc, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&sh->acc_full[slot]);
        tc::mma_commit(&sh->empty[s]);
      }
      // every MMA issued has completed before TMEM is freed
      if (!tc::mma_drain(&sh->mma_done)) failed = true;
    }
  } else {
    // ---------------- epilogue: masked column maxima ----------------
    const int quarter = warp & 3;            // TMEM lanes this warp may touch
    const int key = quarter * 32 + lane;     // key of the block on this thread's lane
    const int et = threadIdx.x - 64;         // 0..127 over the epilogue warps
    int k = 0;
    for (long long it = i0; it < i1; ++it, ++k) {
      const int slot = k % kSlots;
      const int b = int(it / nvis), c = int(it % nvis);
      bool ok = true;
      if (lane == 0) ok = tc::mbar_wait(&sh->acc_full[slot], (k / kSlots) & 1, abort);
      ok = __shfl_sync(MSA_FULL_MASK, ok, 0);
      if (ok) {
        tc::tc_fence_after();
        uint32_t v[N];
#pragma unroll
        for (int h = 0; h < N / 16; ++h)
          tc::tmem_ld16(tmem + (uint32_t(quarter * 32) << 16) + slot * N + h * 16, v + h * 16);
        tc::tmem_ld_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh->acc_empty[slot]);
        const long long j = (long long)c * 128 + key;  // key position in the sequence
#pragma unroll
        for (int n = 0; n < N; ++n) {
          if (n < RG) {
            const bool vis = j <= P.q_pos0 + n / P.Hkv;
            const uint32_t m =
                __reduce_max_sync(MSA_FULL_MASK, vis ? orderable(__uint_as_float(v[n])) : 0u);
            if (lane == 0) sh->red[slot][quarter][n] = m;
          }
        }
      }
      // publishes red[slot]; every epilogue thread leaves together on a failure
      if (epi_any(!ok)) { failed = true; break; }
      if (et < RG) {
        const uint32_t m = max(max(sh->red[slot][0][et], sh->red[slot][1][et]),
                               max(sh->red[slot][2][et], sh->red[slot][3][et]));
        const int i = et / P.Hkv, g = et % P.Hkv;
        // back from the orderable key; 0 means no visible key in the block
        const float val = m == 0u ? -INFINITY
                                  : __uint_as_float((m & 0x80000000u) ? (m & 0x7fffffffu) : ~m);
        if ((long long)c * 128 <= P.q_pos0 + i)
          bmax[((long long)g * P.T + (long long)b * P.Sq + i) * P.nblk + c] = val;
      }
    }
  }
  if (failed) {
    sh->abort = 1;
    atomicOr(status, tc::kStatusWaitTimeout);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

bool index_decode_supported(const Problem& P) {
  const int rg = P.Sq * P.Hkv;
  return !P.f32 && !P.idx4 && P.DI == 128 && P.Bk == 128 && P.Sq <= 8 && rg >= 1 && rg <= kMaxRG &&
         P.kv_rows < (1LL << 31);
}

template <int N, bool FP8>
static cudaError_t launch_n(const CUtensorMap& map, const Problem& P, const void* q_idx,
                            float* bmax, int32_t* status, int nvis, long long items,
                            cudaStream_t s) {
  constexpr size_t smem = smem_bytes<N, FP8>();
  const int grid =
      int(std::min<long long>((long long)sm_count() * Cfg<N, FP8>::kCtasPerSm, items));
  cudaError_t e = cudaFuncSetAttribute(index_decode_kernel<N, FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  index_decode_kernel<N, FP8><<<grid, kThreads, smem, s>>>(
      map, P, static_cast<const uint8_t*>(q_idx), bmax, status, nvis);
  return cudaGetLastError();
}

cudaError_t launch_index_decode(const Problem& P, const void* q_idx, const void* k_idx,
                                float* bmax, int32_t* status, cudaStream_t s) {
  if (!index_decode_supported(P)) return cudaErrorNotSupported;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // k_idx rows of 128 dims as 128-byte-wide boxes of 128 keys (128-byte swizzle)
  CUtensorMap map;
  cuuint64_t dims[2] = {128, cuuint64_t(P.kv_rows)};
  cuuint64_t strides[1] = {P.idx8 ? 128u : 256u};
  cuuint32_t box[2] = {P.idx8 ? 128u : 64u, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, P.idx8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
          const_cast<void*>(k_idx), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int nvis = int((P.q_pos0 + P.Sq - 1) / P.Bk) + 1;
  const long long items = (long long)P.B * nvis;
  const int rg = P.Sq * P.Hkv;
  if (P.idx8)
    return rg <= 16 ? launch_n<16, true>(map, P, q_idx, bmax, status, nvis, items, s)
                    : launch_n<32, true>(map, P, q_idx, bmax, status, nvis, items, s);
  return rg <= 16 ? launch_n<16, false>(map, P, q_idx, bmax, status, nvis, items, s)
                  : launch_n<32, false>(map, P, q_idx, bmax, status, nvis, items, s);
}

}  // namespace msa
