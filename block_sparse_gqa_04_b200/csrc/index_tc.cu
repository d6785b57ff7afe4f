// Index branch on tcgen05 tensor cores: block maxima of the raw index scores
// q_idx . k_idx with the causal mask and the 128-token max-pool fused into the
// epilogue, so no token score ever reaches HBM ("Substantial numerical
// differences with Minimax MSA attention vs Minimax's Reference", section
// 原因分析: amax over each block, per index head; snilld.dk "Hvad er MSA i
// praksis": one index-query head per GQA group, one shared index-key head).
//
// Shapes: bf16 or fp8 (e4m3) index tensors, index_dim 128, block 128, up to 4
// groups.  One persistent CTA per SM walks a contiguous share of the (sequence,
// 128-row query tile, key block) triples that the causal mask leaves, with the
// query tiles in the balanced order of tile_at below.  For each triple and each group one MMA unit
// computes S[128 queries x 128 keys] = q_idx_g . k_idx_block^T in fp32:
//   * TMEM lanes are query rows.  The index queries of the current query tile
//     (all groups, 128 x 128 bf16 each) sit in TMEM columns 0..255 as the A
//     operand, written there once per tile by the epilogue warps;
//   * the k_idx block (128 keys x 128 dims, 32 KB) is the B operand, streamed
//     by TMA (128-byte swizzle) through a 4-stage shared-memory ring and shared
//     by the groups' MMAs, so shared memory only feeds B;
//   * two 128-column fp32 accumulators alternate, so the epilogue of one unit
//     overlaps the MMAs of the next.
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs, warps
// 2-9 load index queries into TMEM and run the epilogue (one query row per
// thread: masked max over the row's 128 columns, one fp32 store per unit).
// The epilogue is two warpgroups, one per accumulator, so that two units drain
// at once while the tensor cores fill the next.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 320;               // TMA, MMA, two epilogue warpgroups
constexpr int kMaxGroups = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 256;           // accumulators follow the A region

// Element type of the index tensors: bf16 (kind::f16, two 64-dim halves per key
// row) or fp8 e4m3 (kind::f8f6f4, one 128-byte half, half the bytes).
template <bool FP8>
struct Idx {
  static constexpr int kRowBytes = FP8 ? 128 : 256;            // one key / query row
  static constexpr int kStageBytes = 128 * kRowBytes;          // one k_idx block
  static constexpr int kHalfBytes = 128 * 128;                 // 128-byte rows x 128 keys
  static constexpr int kSteps = FP8 ? 4 : 8;                   // K steps of 32 bytes
  static constexpr uint32_t kGroupCols = FP8 ? 32 : 64;        // TMEM columns per group
  static constexpr uint32_t kIdesc =
      FP8 ? tc::idesc_e4m3_f32(128, 128) : tc::idesc_bf16_f32(128, 128, 0, 0);
  static constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + 256;
};

// Blocks query tile m (128 rows) of a sequence can see.
__host__ __device__ inline int tile_blocks(const Problem& P, int m) {
  const int last = min(P.Sq - 1, m * 128 + 127);
  return int((P.q_pos0 + last) / P.Bk) + 1;
}

// (tile, block) pairs of one sequence that come before query tile m.  Every
// tile before m is full, so tile m' sees base + m' + 1 blocks.
__host__ __device__ inline long long pairs_before(const Problem& P, int m) {
  const long long base = (P.q_pos0 + 127) / P.Bk;
  return (long long)m * (base + 1) + (long long)m * (m - 1) / 2;
}

__host__ __device__ inline int mtiles(const Problem& P) { return (P.Sq + 127) / 128; }

__host__ __device__ inline long long pairs_per_seq(const Problem& P) {
  const int M = mtiles(P);
  return pairs_before(P, M - 1) + tile_blocks(P, M - 1);
}

// Query tiles are walked in the order 0, M-1, 1, M-2, ... so that every CTA's
// contiguous share of pairs mixes short (early) and long (late) tiles: the
// number of tile switches, each of which reloads the index queries into TMEM,
// is then about the same on every CTA.
__host__ __device__ inline int tile_at(const Problem& P, int u) {
  return (u & 1) ? mtiles(P) - 1 - (u >> 1) : (u >> 1);
}

// Pairs of one sequence before position u of that order: the first (u+1)/2
// tiles plus the last u/2 tiles.
__host__ __device__ inline long long pairs_before_at(const Problem& P, int u, long long per_seq) {
  const int ne = (u + 1) >> 1, no = u >> 1;
  return pairs_before(P, ne) + (no > 0 ? per_seq - pairs_before(P, mtiles(P) - no) : 0);
}

// Walks (b, m, c) over a contiguous range of the linear pair index.
struct Walk {
  int b, u, m, c, nc;
  __device__ void start(const Problem& P, long long L, long long per_seq) {
    b = int(L / per_seq);
    long long l = L % per_seq;
    int lo = 0, hi = mtiles(P) - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (pairs_before_at(P, mid, per_seq) <= l) lo = mid; else hi = mid - 1;
    }
    u = lo;
    m = tile_at(P, u);
    c = int(l - pairs_before_at(P, u, per_seq));
    nc = tile_blocks(P, m);
  }
  // advances; returns true when the next pair starts a new query tile
  __device__ bool next(const Problem& P) {
    if (++c < nc) return false;
    c = 0;
    if (++u == mtiles(P)) { u = 0; ++b; }
    m = tile_at(P, u);
    nc = tile_blocks(P, m);
    return true;
  }
};

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t a_full;
  uint64_t a_empty;
  uint32_t tmem_base;
  int abort;
};

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, Problem P,
                const uint8_t* __restrict__ q_idx, float* __restrict__ bmax,
                int* __restrict__ status, long long per_seq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  using X = Idx<FP8>;
  Bars* bars = reinterpret_cast<Bars*>(smem + kStages * X::kStageBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->acc_full[s], 1);
      tc::mbar_init(&bars->acc_empty[s], 4);
    }
    tc::mbar_init(&bars->a_full, 8);
    tc::mbar_init(&bars->a_empty, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tc::tma_prefetch(&tmap_k);
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const long long total = per_seq * P.B;
  const long long L0 = total * blockIdx.x / gridDim.x;
  const long long L1 = total * (blockIdx.x + 1) / gridDim.x;
  bool failed = false;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && L0 < L1) {
      Walk w;
      w.start(P, L0, per_seq);
      int stage = 0;
      uint32_t phase = 0;
      for (long long L = L0; L < L1; ++L) {
        if (!tc::mbar_wait(&bars->empty[stage], phase ^ 1, abort)) { failed = true; break; }
        tc::mbar_arrive_expect_tx(&bars->full[stage], X::kStageBytes);
        const int row = int(block_row(P, w.b, w.c));
        uint8_t* dst = stages + stage * X::kStageBytes;
        tc::tma_load_2d(dst, &tmap_k, &bars->full[stage], 0, row);
        if (!FP8) tc::tma_load_2d(dst + X::kHalfBytes, &tmap_k, &bars->full[stage], 64, row);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        w.next(P);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && L0 < L1) {
      Walk w;
      w.start(P, L0, per_seq);
      int stage = 0, slot = 0;
      uint32_t phase = 0, acc_phase = 0, a_phase = 0;
      bool seg_start = true;
      for (long long L = L0; L < L1 && !failed; ++L) {
        if (seg_start) {
          if (!tc::mbar_spin(&bars->a_full, a_phase, abort)) { failed = true; break; }
          a_phase ^= 1;
          tc::tc_fence_after();
        }
        if (!tc::mbar_spin(&bars->full[stage], phase, abort)) { failed = true; break; }
        tc::tc_fence_after();
        const uint32_t sbase = tc::smem_addr(stages + stage * X::kStageBytes);
        for (int g = 0; g < P.Hkv; ++g) {
          if (!tc::mbar_spin(&bars->acc_empty[slot], acc_phase ^ 1, abort)) {
            failed = true;
            break;
          }
          tc::tc_fence_after();
          const uint32_t d = tmem + kAccCol + slot * 128;
#pragma unroll
          for (int kk = 0; kk < X::kSteps; ++kk) {
            // 32 bytes of K per step: 16 bf16 or 32 fp8, 8 TMEM columns of A
            const uint64_t bd = tc::sdesc_sw128(sbase + (kk >> 2) * X::kHalfBytes + (kk & 3) * 32,
                                                16, 1024);
            if (FP8)
              tc::mma_ts_f8(d, tmem + g * X::kGroupCols + kk * 8, bd, X::kIdesc, kk > 0 ? 1u : 0u);
            else
              tc::mma_ts(d, tmem + g * X::kGroupCols + kk * 8, bd, X::kIdesc, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&bars->acc_full[slot]);
          slot ^= 1;
          if (slot == 0) acc_phase ^= 1;
        }
        if (failed) break;
        tc::mma_commit(&bars->empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        seg_start = w.next(P);
        if (seg_start || L + 1 == L1) tc::mma_commit(&bars->a_empty);
      }
    }
  } else {
    // ---------------- index-query loader + epilogue (two warpgroups) ----------------
    const int ewg = (warp - 2) >> 2;        // accumulator slot this warpgroup drains
    const int quarter = warp & 3;           // TMEM lanes this warp may touch
    const int row = quarter * 32 + lane;    // query row inside the tile
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    if (L0 < L1) {
      Walk w;
      w.start(P, L0, per_seq);
      uint32_t ae_phase = 0;
      int k = 0;                            // unit counter, the same on every warp
      bool seg_start = true, first = true;
      for (long long L = L0; L < L1 && !failed; ++L) {
        const int i = w.m * 128 + row;      // query index inside the sequence
        const bool valid = i < P.Sq;
        const long long r = (long long)w.b * P.Sq + i;
        if (seg_start) {
          if (!first) {
            if (!__all_sync(MSA_FULL_MASK, tc::mbar_wait(&bars->a_empty, ae_phase, abort))) {
              failed = true;
              break;
            }
            ae_phase ^= 1;
            tc::tc_fence_after();
          }
          first = false;
          // each warpgroup writes the index queries of every other group
          const uint4* src = reinterpret_cast<const uint4*>(q_idx + r * P.Hkv * X::kRowBytes);
          for (int g = ewg; g < P.Hkv; g += 2) {
#pragma unroll
            for (int h = 0; h < X::kRowBytes / 128; ++h) {
              uint32_t v[32];
#pragma unroll
              for (int x = 0; x < 8; ++x) {
                uint4 u = valid ? __ldg(src + g * (X::kRowBytes / 16) + h * 8 + x)
                                : make_uint4(0, 0, 0, 0);
                v[4 * x + 0] = u.x;
                v[4 * x + 1] = u.y;
                v[4 * x + 2] = u.z;
                v[4 * x + 3] = u.w;
              }
              tc::tmem_st32(tmem + lane_addr + g * X::kGroupCols + h * 32, v);
            }
          }
          tc::tmem_st_wait();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->a_full);
        }
        const long long t = P.q_pos0 + i;
        const long long lim = t - (long long)w.c * P.Bk;  // last visible column
        for (int g = 0; g < P.Hkv; ++g, ++k) {
          if ((k & 1) != ewg) continue;     // the other warpgroup's unit
          const uint32_t par = (k >> 1) & 1;
          if (!__all_sync(MSA_FULL_MASK, tc::mbar_wait(&bars->acc_full[ewg], par, abort))) {
            failed = true;
            break;
          }
          tc::tc_fence_after();
          // all 128 columns in flight at once, then a tree of maxima (eight
          // independent chains) instead of one 128-long dependent chain
          uint32_t v[4][32];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc::tmem_ld32(tmem + lane_addr + kAccCol + ewg * 128 + j * 32, v[j]);
          tc::tmem_ld_wait();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->acc_empty[ewg]);
          float mx[8];
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = -INFINITY;
          if (__all_sync(MSA_FULL_MASK, lim >= 127)) {
#pragma unroll
            for (int x = 0; x < 128; ++x)
              mx[x & 7] = fmaxf(mx[x & 7], __uint_as_float(v[x >> 5][x & 31]));
          } else {
#pragma unroll
            for (int x = 0; x < 128; ++x)
              if (x <= lim) mx[x & 7] = fmaxf(mx[x & 7], __uint_as_float(v[x >> 5][x & 31]));
          }
          const float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
          if (valid) bmax[((long long)g * P.T + r) * P.nblk + w.c] = m;
        }
        seg_start = w.next(P);
      }
    }
  }
  if (failed) {
    bars->abort = 1;
    atomicOr(status, tc::kStatusWaitTimeout);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
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

bool index_tc_supported(const Problem& P) {
  return !P.f32 && P.DI == 128 && P.Bk == 128 && P.Hkv <= kMaxGroups && P.Sq > 8 &&
         P.kv_rows < (1LL << 31);
}

template <bool FP8>
static cudaError_t launch_t(const Problem& P, const void* q_idx, const void* k_idx, float* bmax,
                           int32_t* status, cudaStream_t s) {
  using X = Idx<FP8>;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // k_idx rows of 128 dims, copied as 128-byte-wide boxes of 128 keys (128-byte swizzle)
  CUtensorMap map;
  cuuint64_t dims[2] = {FP8 ? 128u : 128u, cuuint64_t(P.kv_rows)};
  cuuint64_t strides[1] = {cuuint64_t(X::kRowBytes)};
  cuuint32_t box[2] = {FP8 ? 128u : 64u, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(k_idx), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const long long per_seq = pairs_per_seq(P);
  const long long total = per_seq * P.B;
  const int grid = int(std::min<long long>(sm_count(), total));
  cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(X::kSmemBytes));
  if (e != cudaSuccess) return e;
  index_tc_kernel<FP8><<<grid, kThreads, X::kSmemBytes, s>>>(
      map, P, static_cast<const uint8_t*>(q_idx), bmax, status, per_seq);
  return cudaGetLastError();
}

cudaError_t launch_index_tc(const Problem& P, const void* q_idx, const void* k_idx,
                            float* bmax, int32_t* status, cudaStream_t s) {
  return P.idx8 ? launch_t<true>(P, q_idx, k_idx, bmax, status, s)
                : launch_t<false>(P, q_idx, k_idx, bmax, status, s);
}

}  // namespace msa
