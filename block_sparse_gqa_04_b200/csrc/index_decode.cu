// Index branch for a few query rows per sequence (decode): block maxima of the
// raw index scores q_idx . k_idx over the visible tokens of every 128-token
// block ("Substantial numerical differences with Minimax MSA attention vs
// Minimax's Reference", section 原因分析: amax over each block, per index
// head; snilld.dk "Hvad er MSA i praksis": one index-query head per GQA group,
// one shared index-key head).
//
// With one query per sequence the work is a stream over k_idx (0.25 KB per key)
// with a handful of dot products per key, so it is bound by HBM, not by any
// arithmetic unit.  Persistent CTAs stream contiguous ranges of (sequence,
// block) items of 32 KB through a ring of shared-memory stages filled by TMA (128-byte swizzle, which
// also makes each thread's 16-byte reads of its own key row conflict-free).
// Two teams of four warps take alternate items; in a team, thread k owns key k
// of the block and forms its dot products with every (row, group) index query
// (packed fp32x2 FMAs against queries broadcast from shared memory); the
// block maximum per (row, group) is a warp redux plus a max over the four
// warps.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kStages = 5;
constexpr int kBlkBytes = 128 * 128 * 2;   // one block of k_idx
constexpr int kHalfBytes = kBlkBytes / 2;
constexpr int kTeamThreads = 128;
constexpr int kThreads = 2 * kTeamThreads + 32;  // two teams + a producer warp
constexpr int kMaxRG = 16;                 // (rows per sequence) x groups handled

struct Shared {
  uint64_t full[kStages], empty[kStages];
  float q[2][kMaxRG][128];                 // per team: index queries of its sequence, fp32
  uint32_t red[2][4][kMaxRG];              // per team: warp maxima (orderable keys)
  int abort;
};

constexpr size_t kSmemBytes = 1024 + kStages * kBlkBytes + sizeof(Shared) + 64;
static_assert(kSmemBytes <= 232448, "more dynamic shared memory than a B200 CTA can have");

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ void team_sync(int team) {
  asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(kTeamThreads) : "memory");
}

// Team barrier that also returns whether any thread of the team passed `v`.
__device__ __forceinline__ bool team_any(int team, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(team + 1), "r"(kTeamThreads)
      : "memory");
  return r != 0;
}

// RG = (query rows per sequence) x groups, fixed at compile time so that only
// the live dot products are formed.
template <int RG>
__global__ void __launch_bounds__(kThreads, 1)
index_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, Problem P,
                    const __nv_bfloat16* __restrict__ q_idx, float* __restrict__ bmax,
                    int* __restrict__ status, int nvis) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  Shared* sh = reinterpret_cast<Shared*>(smem + kStages * kBlkBytes);
  volatile int* abort = &sh->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&sh->full[s], 1);
      tc::mbar_init(&sh->empty[s], 4);  // the four warps of the team that used it
    }
    sh->abort = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  // each CTA streams a contiguous range of (sequence, block) items, so it stays
  // on one sequence's index queries and reads consecutive blocks
  const long long items = (long long)P.B * nvis;
  const long long i0 = items * blockIdx.x / gridDim.x;
  const long long i1 = items * (blockIdx.x + 1) / gridDim.x;
  bool failed = false;
  if (warp == 8) {
    // ---------------- producer ----------------
    if (lane == 0) {
      tc::tma_prefetch(&tmap_k);
      int k = 0;
      for (long long it = i0; it < i1; ++it, ++k) {
        const int s = k % kStages;
        if (!tc::mbar_wait(&sh->empty[s], ((k / kStages) & 1) ^ 1, abort)) { failed = true; break; }
        const int b = int(it / nvis), c = int(it % nvis);
        tc::mbar_arrive_expect_tx(&sh->full[s], kBlkBytes);
        const int row = b * P.Skv + c * 128;
        tc::tma_load_2d(stages + s * kBlkBytes, &tmap_k, &sh->full[s], 0, row);
        tc::tma_load_2d(stages + s * kBlkBytes + kHalfBytes, &tmap_k, &sh->full[s], 64, row);
      }
    }
  } else {
    // ---------------- teams ----------------
    const int team = warp >> 2, kw = warp & 3;
    const int key = kw * 32 + lane;          // key of the block this thread owns
    int qb = -1;                             // sequence whose queries sit in sh->q[team]
    int k = team;
    for (long long it = i0 + team; it < i1; it += 2, k += 2) {
      const int s = k % kStages;
      const int b = int(it / nvis), c = int(it % nvis);
      if (b != qb) {
        team_sync(team);
        for (int e = threadIdx.x - team * kTeamThreads; e < RG * 128; e += kTeamThreads)
          sh->q[team][e >> 7][e & 127] =
              __bfloat162float(q_idx[(long long)b * RG * 128 + e]);
        team_sync(team);
        qb = b;
      }
      // the whole team gives up together, so no warp is left at a team barrier
      if (team_any(team, !tc::mbar_wait(&sh->full[s], (k / kStages) & 1, abort))) {
        failed = true;
        break;
      }
      const uint8_t* kr = stages + s * kBlkBytes + key * 128;
      uint64_t acc[RG];
#pragma unroll
      for (int x = 0; x < RG; ++x) acc[x] = 0;
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {
        // 16-byte chunk j of this key: half j / 8, swizzled position (j % 8) ^ (key % 8)
        const uint4 u = *reinterpret_cast<const uint4*>(kr + (j >> 3) * kHalfBytes +
                                                        (((j & 7) ^ (key & 7)) << 4));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint64_t kp[4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
          kp[x] = (uint64_t(w[x] & 0xffff0000u) << 32) | uint64_t(w[x] << 16);
#pragma unroll
        for (int x = 0; x < RG; ++x) {
          const uint4* qp = reinterpret_cast<const uint4*>(&sh->q[team][x][8 * j]);
          const uint4 q0 = qp[0], q1 = qp[1];
          acc[x] = fma2(kp[0], (uint64_t(q0.y) << 32) | q0.x, acc[x]);
          acc[x] = fma2(kp[1], (uint64_t(q0.w) << 32) | q0.z, acc[x]);
          acc[x] = fma2(kp[2], (uint64_t(q1.y) << 32) | q1.x, acc[x]);
          acc[x] = fma2(kp[3], (uint64_t(q1.w) << 32) | q1.z, acc[x]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh->empty[s]);  // this warp is done with the stage
      const long long j = (long long)c * 128 + key;    // key position in the sequence
#pragma unroll
      for (int x = 0; x < RG; ++x) {
        const int i = x / P.Hkv;
        const bool vis = j < P.Skv && j <= P.q_pos0 + i;
        const float sc = __uint_as_float(uint32_t(acc[x])) + __uint_as_float(uint32_t(acc[x] >> 32));
        const uint32_t m = __reduce_max_sync(MSA_FULL_MASK, vis ? orderable(sc) : 0u);
        if (lane == 0) sh->red[team][kw][x] = m;
      }
      team_sync(team);
      const int t = threadIdx.x - team * kTeamThreads;
      if (t < RG) {
        const uint32_t m = max(max(sh->red[team][0][t], sh->red[team][1][t]),
                               max(sh->red[team][2][t], sh->red[team][3][t]));
        const int i = t / P.Hkv, g = t % P.Hkv;
        // back from the orderable key; 0 means no visible key in the block
        const float v = m == 0u ? -INFINITY
                                : __uint_as_float((m & 0x80000000u) ? (m & 0x7fffffffu) : ~m);
        if ((long long)c * 128 <= P.q_pos0 + i)
          bmax[((long long)g * P.T + (long long)b * P.Sq + i) * P.nblk + c] = v;
      }
      team_sync(team);  // red[] is reused by the next item
    }
  }
  if (failed) {
    sh->abort = 1;
    atomicOr(status, tc::kStatusWaitTimeout);
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

// (rows per sequence) x groups: the widths the kernel is instantiated for
static int rg_width(const Problem& P) {
  const int rg = P.Sq * P.Hkv;
  return (rg == 4 || rg == 8 || rg == 16) ? rg : 0;
}

bool index_decode_supported(const Problem& P) {
  return !P.f32 && P.DI == 128 && P.Bk == 128 && P.Sq <= 8 && rg_width(P) != 0 &&
         (long long)P.B * P.Skv < (1LL << 31);
}

cudaError_t launch_index_decode(const Problem& P, const void* q_idx, const void* k_idx,
                                float* bmax, int32_t* status, cudaStream_t s) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  cuuint64_t dims[2] = {128, cuuint64_t(P.B) * P.Skv};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k_idx), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int nvis = int((P.q_pos0 + P.Sq - 1) / P.Bk) + 1;
  const long long items = (long long)P.B * nvis;
  const int grid = int(std::min<long long>(sm_count(), (items + 1) / 2));
  auto kern = index_decode_kernel<4>;
  switch (P.Sq * P.Hkv) {
    case 4: kern = index_decode_kernel<4>; break;
    case 8: kern = index_decode_kernel<8>; break;
    case 16: kern = index_decode_kernel<16>; break;
    default: return cudaErrorNotSupported;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemBytes));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(map, P, static_cast<const __nv_bfloat16*>(q_idx), bmax,
                                          status, nvis);
  return cudaGetLastError();
}

}  // namespace msa
