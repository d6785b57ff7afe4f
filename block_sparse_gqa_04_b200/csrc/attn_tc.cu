// Main branch on tcgen05 tensor cores: KV-outer block-sparse attention with
// query gather ("MiniMax 稀疏注意力" (hyper.ai), sections 摘要 and 核心贡献:
// exp-free top-k plus KV-outer sparse attention to keep the tensor cores busy
// under block-granular access; section 引言: the FlashAttention loop order is
// swapped; snilld.dk "Hvad er MSA i praksis": every query head of a group
// attends over the causally visible tokens of the group's selected blocks).
//
// Shapes: bf16, head_dim 128, 16 query heads per group, block 128.  The work is
// the flat list of 128-row tiles that the block -> query lists define: a tile is
// 8 gathered queries x 16 heads of one (sequence, group, query chunk, block).
// One persistent CTA per SM takes a contiguous share of the tiles.  Per tile:
//   * TMA loads the block's K and V (128 keys x 128 dims each, 128-byte swizzle)
//     into one of two buffers, once per list, and gathers the 8 queries' Q rows
//     (16 heads x 128 dims, contiguous in memory) with two boxes per query;
//   * S = Q K^T (both K-major in shared memory) lands in TMEM, one row per lane;
//   * the softmax warps read their row, apply the scale and the causal cut of
//     the local block, and write P (bf16) back over S in TMEM;
//   * O = P V runs with P from TMEM and V as an MN-major shared-memory operand;
//   * the softmax warps normalise O by the row sum, stage the bf16 rows in
//     shared memory and bulk-store them (each warp its own 32 rows, which are
//     contiguous in the entry-ordered partial states); the base-2
//     log-normaliser goes with them.
// TMEM holds two (S|P, O) buffers of 256 columns, so the S MMA of the next tile
// runs while the softmax of this one is computed.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kThreads = 192;                 // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr int kRows = 128;
constexpr int kQBytes = kRows * 128 * 2;      // 32 KB: 128 rows x 128 dims
constexpr int kQHalf = kQBytes / 2;           // one 64-dim half
constexpr int kKVBytes = 2 * kQBytes;         // K then V
constexpr int kOutBytes = kRows * 128 * 2;    // staging of one tile's bf16 rows
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescS = tc::idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, 128, 0, 1);  // V is MN-major
constexpr int kGroup = 16;                    // query heads per group
constexpr int kQPerTile = kRows / kGroup;     // 8 gathered queries

struct Bars {
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2], o_full[2], buf_empty[2];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 + 2 * kQBytes + 2 * kKVBytes + kOutBytes + 256;

__device__ __forceinline__ long long find_list(const int32_t* __restrict__ tile_off,
                                               long long nlists, int tile) {
  long long lo = 0, hi = nlists;  // tile_off[lo] <= tile < tile_off[hi]
  while (hi - lo > 1) {
    long long mid = (lo + hi) >> 1;
    if (__ldg(tile_off + mid) <= tile) lo = mid; else hi = mid;
  }
  return lo;
}

// Walks the tiles [t0, t1) in order, tracking the list each one belongs to.
struct TileWalk {
  const Problem* P;
  const int32_t* tile_off;
  const int32_t* list_off;
  int tile, t1;
  long long lid;
  int c, g, b, e0, n;
  bool new_list;
  __device__ void decode() {
    c = int(lid % P->nblk);
    const long long rest = lid / P->nblk;
    g = int((rest / P->nqc) % P->Hkv);
    b = int(rest / ((long long)P->nqc * P->Hkv));
    e0 = __ldg(list_off + lid) + (tile - __ldg(tile_off + lid)) * kQPerTile;
    n = min(kQPerTile, __ldg(list_off + lid + 1) - e0);
  }
  __device__ void start(const Problem& Pr, const Lists& L, int a, int z) {
    P = &Pr;
    tile_off = L.tile_off;
    list_off = L.list_off;
    tile = a;
    t1 = z;
    lid = find_list(tile_off, Pr.nlists, a);
    new_list = true;
    decode();
  }
  // true if the tile after this one (in range) belongs to another list
  __device__ bool last_of_list() const {
    return tile + 1 >= t1 || tile + 1 >= __ldg(tile_off + lid + 1);
  }
  __device__ void next() {
    ++tile;
    new_list = false;
    while (tile >= __ldg(tile_off + lid + 1)) {
      ++lid;
      new_list = true;
    }
    decode();
  }
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(MSA_FULL_MASK, tc::mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
               const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v,
               const __grid_constant__ CUtensorMap tmap_o32,
               const __grid_constant__ CUtensorMap tmap_o16, Problem P, Lists L,
               __nv_bfloat16* __restrict__ part_o, float* __restrict__ part_lse,
               int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = smem;                          // [2][32 KB]
  uint8_t* kvbuf = qbuf + 2 * kQBytes;           // [2][K 32 KB | V 32 KB]
  uint8_t* obuf = kvbuf + 2 * kKVBytes;          // 32 KB staging
  Bars* bars = reinterpret_cast<Bars*>(obuf + kOutBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 1);
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 4);
      tc::mbar_init(&bars->o_full[s], 1);
      tc::mbar_init(&bars->buf_empty[s], 4);
    }
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch(&tmap_q);
    tc::tma_prefetch(&tmap_k);
    tc::tma_prefetch(&tmap_v);
    tc::tma_prefetch(&tmap_o32);
    tc::tma_prefetch(&tmap_o16);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int total = __ldg(L.tile_off + P.nlists);
  const int t0 = int((long long)total * blockIdx.x / gridDim.x);
  const int t1 = int((long long)total * (blockIdx.x + 1) / gridDim.x);
  bool failed = false;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && t0 < t1) {
      TileWalk w;
      w.start(P, L, t0, t1);
      int kv_stage = 0, q_stage = 0;
      uint32_t kv_phase = 0, q_phase = 0;
      for (int i = t0; i < t1; ++i) {
        if (w.new_list) {
          if (!tc::mbar_wait(&bars->kv_empty[kv_stage], kv_phase ^ 1, abort)) {
            failed = true;
            break;
          }
          uint64_t* fb = &bars->kv_full[kv_stage];
          tc::mbar_arrive_expect_tx(fb, kKVBytes);
          uint8_t* dst = kvbuf + kv_stage * kKVBytes;
          const int key0 = w.b * P.Skv + w.c * P.Bk;
          tc::tma_load_3d(dst, &tmap_k, fb, 0, w.g, key0);
          tc::tma_load_3d(dst + kQHalf, &tmap_k, fb, 64, w.g, key0);
          tc::tma_load_3d(dst + kQBytes, &tmap_v, fb, 0, w.g, key0);
          tc::tma_load_3d(dst + kQBytes + kQHalf, &tmap_v, fb, 64, w.g, key0);
          kv_stage ^= 1;
          if (kv_stage == 0) kv_phase ^= 1;
        }
        if (!tc::mbar_wait(&bars->q_empty[q_stage], q_phase ^ 1, abort)) {
          failed = true;
          break;
        }
        int rows[kQPerTile];
#pragma unroll
        for (int e = 0; e < kQPerTile; ++e)
          rows[e] = e < w.n ? (__ldg(L.entries + w.e0 + e) >> 5) : 0;
        uint64_t* fb = &bars->q_full[q_stage];
        tc::mbar_arrive_expect_tx(fb, uint32_t(w.n) * 2 * kGroup * 128);
        uint8_t* dst = qbuf + q_stage * kQBytes;
#pragma unroll
        for (int e = 0; e < kQPerTile; ++e) {
          if (e < w.n) {
            const int qrow = rows[e] * P.Hq + w.g * kGroup;
            tc::tma_load_2d(dst + e * (kGroup * 128), &tmap_q, fb, 0, qrow);
            tc::tma_load_2d(dst + kQHalf + e * (kGroup * 128), &tmap_q, fb, 64, qrow);
          }
        }
        q_stage ^= 1;
        if (q_stage == 0) q_phase ^= 1;
        if (i + 1 < t1) w.next();
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && t0 < t1) {
      TileWalk w;
      w.start(P, L, t0, t1);
      int kv_stage = 0, q_stage = 0;
      uint32_t kv_phase = 0, q_phase = 0;
      int tile_kv[2] = {0, 0};
      bool tile_last[2] = {false, false};
      // issues S = Q K^T of tile i into buffer i & 1
      auto issue_s = [&](int i) -> bool {
        const int buf = i & 1;
        if (w.new_list) {
          if (!tc::mbar_wait(&bars->kv_full[kv_stage], kv_phase, abort)) return false;
          tile_kv[buf] = kv_stage;
          kv_stage ^= 1;
          if (kv_stage == 0) kv_phase ^= 1;
        } else {
          tile_kv[buf] = tile_kv[buf ^ 1];
        }
        tile_last[buf] = w.last_of_list();
        if (!tc::mbar_wait(&bars->q_full[q_stage], q_phase, abort)) return false;
        if (!tc::mbar_wait(&bars->buf_empty[buf], (((i - t0) >> 1) & 1) ^ 1, abort)) return false;
        tc::tc_fence_after();
        const uint32_t qa = tc::smem_addr(qbuf + q_stage * kQBytes);
        const uint32_t ka = tc::smem_addr(kvbuf + tile_kv[buf] * kKVBytes);
        const uint32_t d = tmem + buf * 256;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kQHalf + (kk & 3) * 32;
          tc::mma_ss(d, tc::sdesc_sw128(qa + off, 16, 1024), tc::sdesc_sw128(ka + off, 16, 1024),
                     kIdescS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->s_full[buf]);
        tc::mma_commit(&bars->q_empty[q_stage]);
        q_stage ^= 1;
        if (q_stage == 0) q_phase ^= 1;
        return true;
      };
      if (!issue_s(t0)) failed = true;
      for (int i = t0; i < t1 && !failed; ++i) {
        const int buf = i & 1;
        const int kvs = tile_kv[buf];
        const bool last = tile_last[buf];
        if (i + 1 < t1) {
          w.next();
          if (!issue_s(i + 1)) { failed = true; break; }
        }
        if (!tc::mbar_wait(&bars->p_full[buf], ((i - t0) >> 1) & 1, abort)) { failed = true; break; }
        tc::tc_fence_after();
        const uint32_t va = tc::smem_addr(kvbuf + kvs * kKVBytes + kQBytes);
        const uint32_t o = tmem + buf * 256 + 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          tc::mma_ts(o, tmem + buf * 256 + kk * 8, tc::sdesc_sw128(va + kk * 2048, kQHalf, 1024),
                     kIdescO, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars->o_full[buf]);
        if (last) tc::mma_commit(&bars->kv_empty[kvs]);
      }
    }
  } else {
    // ---------------- softmax + epilogue ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    const float sl2 = P.scale * 1.4426950408889634f;
    if (t0 < t1) {
      TileWalk w;
      w.start(P, L, t0, t1);
      for (int i = t0; i < t1; ++i) {
        const int buf = i & 1;
        const uint32_t par = ((i - t0) >> 1) & 1;
        const int el = row / kGroup, hh = row % kGroup;
        const bool valid = el < w.n;
        const int packed = valid ? __ldg(L.entries + w.e0 + el) : 0;
        const int r = packed >> 5;
        const long long t = P.q_pos0 + r % P.Sq;
        const int lim = int(min(127LL, t - (long long)w.c * P.Bk));  // last visible column
        if (!warp_wait(&bars->s_full[buf], par, abort)) { failed = true; break; }
        tc::tc_fence_after();
        float s[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t v[32];
          tc::tmem_ld32(tmem + lane_addr + buf * 256 + j * 32, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) s[j * 32 + x] = __uint_as_float(v[x]);
        }
        float m = -INFINITY;
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x <= lim) m = fmaxf(m, s[x]);
        const float ms = m * sl2;
        float l = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int c0 = 64 * h + 2 * x;
            const float p0 = c0 <= lim ? exp2f(fmaf(s[c0], sl2, -ms)) : 0.f;
            const float p1 = c0 + 1 <= lim ? exp2f(fmaf(s[c0 + 1], sl2, -ms)) : 0.f;
            l += p0 + p1;
            v[x] = pack_bf16(p0, p1);
          }
          tc::tmem_st32(tmem + lane_addr + buf * 256 + h * 32, v);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->p_full[buf]);
        if (!warp_wait(&bars->o_full[buf], par, abort)) { failed = true; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t v[32];
          tc::tmem_ld32(tmem + lane_addr + buf * 256 + 128 + j * 32, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) s[j * 32 + x] = __uint_as_float(v[x]);
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->buf_empty[buf]);
        // Stage the normalised bf16 row.  Each warp owns 32 consecutive rows (two
        // gathered queries, contiguous in the entry-ordered partial states) and
        // stores them itself with TMA, so the epilogue needs no barrier across
        // warps.  The staging uses the 128-byte swizzle (16-byte chunk j of a
        // row goes to chunk j ^ (row % 8)), which the TMA store undoes.
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        __syncwarp();
        const float inv = 1.f / l;
        uint8_t* wst = obuf + quarter * 8192;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c0 = 64 * h + 8 * j;
            uint4 u;
            u.x = pack_bf16(s[c0 + 0] * inv, s[c0 + 1] * inv);
            u.y = pack_bf16(s[c0 + 2] * inv, s[c0 + 3] * inv);
            u.z = pack_bf16(s[c0 + 4] * inv, s[c0 + 5] * inv);
            u.w = pack_bf16(s[c0 + 6] * inv, s[c0 + 7] * inv);
            *reinterpret_cast<uint4*>(wst + h * 4096 + lane * 128 + ((j ^ (lane & 7)) << 4)) = u;
          }
        }
        if (valid) part_lse[(long long)(w.e0 + el) * kGroup + hh] = ms + log2f(l);
        tc::fence_async_smem();
        __syncwarp();
        const int nrows = min(32, w.n * kGroup - quarter * 32);  // 0, 16 or 32
        if (lane == 0 && nrows > 0) {
          const CUtensorMap* map = nrows == 32 ? &tmap_o32 : &tmap_o16;
          const int grow = w.e0 * kGroup + quarter * 32;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            asm volatile(
                "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                    reinterpret_cast<uint64_t>(map)),
                "r"(64 * h), "r"(grow), "r"(tc::smem_addr(wst + h * 4096))
                : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (i + 1 < t1) w.next();
      }
      if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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

bool attn_tc_supported(const Problem& P) {
  return !P.f32 && P.D == 128 && P.G == kGroup && P.Bk == 128 &&
         (long long)P.T * P.Hq < (1LL << 31) && (long long)P.B * P.Skv < (1LL << 31);
}

cudaError_t launch_attn_tc(const Problem& P, const void* q, const void* k, const void* v,
                           const Lists& L, const Partials& part, int32_t* status,
                           cudaStream_t s) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mo32, mo16;
  {
    cuuint64_t dims[2] = {128, cuuint64_t(P.T) * P.Hq};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, kGroup};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {128, cuuint64_t(P.Hkv), cuuint64_t(P.B) * P.Skv};
    cuuint64_t strides[2] = {128 * 2, cuuint64_t(P.Hkv) * 128 * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // partial states: [entries * 16 rows, 128 dims] bf16, stored 16 or 32 rows at a time
    cuuint64_t dims[2] = {128, cuuint64_t(P.T) * P.Hq * P.K};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t estr[2] = {1, 1};
    cuuint32_t box32[2] = {64, 32}, box16[2] = {64, 16};
    if (enc(&mo32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, part.o, dims, strides, box32, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (enc(&mo16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, part.o, dims, strides, box16, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemBytes));
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<sm_count(), kThreads, kSmemBytes, s>>>(
      mq, mk, mv, mo32, mo16, P, L, static_cast<__nv_bfloat16*>(part.o), part.lse2, status);
  return cudaGetLastError();
}

}  // namespace msa
