// Exp-free top-k block selection, one warp per (GQA group, query row).
//
// snilld.dk "Hvad er MSA i praksis": each query keeps k blocks per GQA group
// and its own block is always kept; section "Teknisk forklaring hvorfor
// kompleksiteten skifter": softmax preserves the order, so raw block scores are
// ranked and no exponential is taken.  "Substantial numerical differences ...",
// section 解决步骤: boost and top-k act per index head, never pooled across
// heads.  The local block floor(t/Bk) takes one of the k slots; the other
// min(k, visible) - 1 slots go to the earlier blocks with the largest keys
// (score, then lower block id); ids are written ascending, -1 padded.
//
// Selection runs in two phases.  Phase 1 takes each lane's largest key over its
// strided share of the row and finds the `need`-th largest of those 32 lane
// maxima, tau: the lanes holding the top `need` maxima give `need` distinct keys
// >= tau, so the true top-`need` keys are all >= tau.  The keys >= tau (a few
// dozen on typical rows) are compacted into shared memory.  Phase 2 keeps the
// `need` largest of them.  Keys are unique (they carry the block id), so a key's
// rank (how many keys are larger) decides both steps: each lane counts the
// larger keys among the 32 it sees through shuffles, which are independent of
// one another, instead of running `need` dependent warp-wide maxima.  Rows with
// more than 32 candidates pick them one warp-wide maximum at a time (each pass
// takes the largest key below the previous pick), and rows with more than fit in
// shared memory rescan the row for each pass.  Only the set matters: the kept
// ids are written in ascending order.
#include "common.cuh"
#include "internal.h"

namespace msa {

constexpr int kTopkWarps = 8;
constexpr int kCandCap = 128;  // candidates >= tau kept in shared memory per warp

// Number of lanes among 0 .. n-1 whose key is larger than this lane's.
__device__ __forceinline__ int warp_rank_u64(uint64_t v, int n) {
  const uint32_t hi = uint32_t(v >> 32), lo = uint32_t(v);
  int r = 0;
#pragma unroll 8
  for (int i = 0; i < n; ++i) {
    const uint32_t oh = __shfl_sync(MSA_FULL_MASK, hi, i);
    const uint32_t ol = __shfl_sync(MSA_FULL_MASK, lo, i);
    r += (oh > hi) || (oh == hi && ol > lo);
  }
  return r;
}

// LISTS: one query row per sequence and every row keeps top_k blocks, so each
// block -> query list holds at most one entry and the lists are the identity
// layout (entry = (group, row, slot)); the kernel then also writes the entries,
// their positions and the one-query tile records the attention kernel reads,
// in place of the separate list kernel.
template <bool LISTS>
__global__ void __launch_bounds__(256) topk_kernel(Problem P, const float* __restrict__ bmax,
                                                   int32_t* __restrict__ q2k, Lists L) {
  __shared__ uint64_t cand_all[kTopkWarps][kCandCap];
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const long long wid = (long long)blockIdx.x * kTopkWarps + w;
  if (wid >= (long long)P.Hkv * P.T) return;
  uint64_t* cand = cand_all[w];
  const int g = int(wid / P.T);
  const int r = int(wid % P.T);
  const long long t = P.q_pos0 + r % P.Sq;
  const int c_t = int(t / P.Bk);
  const int ksel = min(P.K, c_t + 1);
  const int need = ksel - 1;  // earlier blocks to pick
  int mine = INT_MAX;         // lanes 0 .. need-1 hold the picks
  if (need == c_t) {
    // every visible block is selected
    if (lane < c_t) mine = lane;
  } else if (need > 0) {
    const float* row = bmax + ((long long)g * P.T + r) * P.nblk;
    // phase 1: lane maxima, and tau = the need-th largest of them
    uint64_t lmax = 0;
    for (int c = lane; c < c_t; c += 32) {
      uint64_t key = block_key(row[c], c);
      lmax = key > lmax ? key : lmax;
    }
    // lanes without a block hold 0 and rank below every real key; since
    // need < c_t, the lane of rank need - 1 holds a real key
    const int r1 = warp_rank_u64(lmax, 32);
    const int src = __ffs(__ballot_sync(MSA_FULL_MASK, r1 == need - 1)) - 1;
    const uint64_t tau = (uint64_t(__shfl_sync(MSA_FULL_MASK, uint32_t(lmax >> 32), src)) << 32) |
                         __shfl_sync(MSA_FULL_MASK, uint32_t(lmax), src);
    // compact the keys >= tau
    int count = 0;
    for (int base = 0; base < c_t; base += 32) {
      const int c = base + lane;
      const uint64_t key = c < c_t ? block_key(row[c], c) : 0;
      const bool take = key >= tau;
      const unsigned m = __ballot_sync(MSA_FULL_MASK, take);
      const int pos = count + __popc(m & ((1u << lane) - 1u));
      if (take && pos < kCandCap) cand[pos] = key;
      count += __popc(m);
    }
    __syncwarp();
    if (count <= 32) {
      // phase 2 by rank: keep the candidates with fewer than `need` larger
      // ones, placed in lanes 0 .. need-1 by their rank
      const uint64_t key = lane < count ? cand[lane] : 0;
      const int r2 = warp_rank_u64(key, count);
      __syncwarp();
      if (lane < count && r2 < need) cand[r2] = key;
      __syncwarp();
      if (lane < need) mine = key_block(cand[lane]);
    } else {
      // phase 2: `need` passes, each taking the largest key below the last pick
      uint64_t prev = ~0ull;
      for (int s = 0; s < need; ++s) {
        uint64_t best = 0;
        if (count <= kCandCap) {
          for (int e = lane; e < count; e += 32) {
            const uint64_t key = cand[e];
            if (key < prev && key > best) best = key;
          }
        } else {
          for (int c = lane; c < c_t; c += 32) {
            const uint64_t key = block_key(row[c], c);
            if (key >= tau && key < prev && key > best) best = key;
          }
        }
        best = warp_max_u64(best);
        if (lane == s) mine = key_block(best);
        prev = best;
      }
    }
  }
  if (lane == need) mine = c_t;
  const int sorted = warp_sort_asc(mine);
  if (lane < P.K) q2k[((long long)g * P.T + r) * P.K + lane] = lane < ksel ? sorted : -1;
  if (LISTS && lane < P.K) {
    const int e = int(((long long)g * P.T + r) * P.K + lane);  // ksel == K on every row
    L.entries[e] = (r << 5) | lane;
    L.pos[e] = e;
    TileRec rec;
    rec.c = sorted;
    rec.g = g;
    rec.b = r / P.Sq;
    rec.e0 = e;
    rec.n = 1;
    rec.tend = e + 1;
    rec.lid = e;
    rec.pad = 0;
    rec.rows[0] = r;
#pragma unroll
    for (int x = 1; x < 8; ++x) rec.rows[x] = 0;
    reinterpret_cast<TileRec*>(L.tiles)[e] = rec;
    if (wid == 0 && lane == 0) L.tile_off[P.nlists] = P.Hkv * P.T * P.K;
  }
}

cudaError_t launch_topk(const Problem& P, const float* bmax, int32_t* q2k, cudaStream_t s) {
  long long warps = (long long)P.Hkv * P.T;
  if (warps == 0) return cudaSuccess;
  long long blocks = (warps + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<false><<<unsigned(blocks), 32 * kTopkWarps, 0, s>>>(P, bmax, q2k, Lists{});
  return cudaGetLastError();
}

bool topk_writes_lists(const Problem& P) {
  return lists_direct(P) && P.q_pos0 >= (long long)(P.K - 1) * P.Bk;
}

cudaError_t launch_topk_lists(const Problem& P, const float* bmax, int32_t* q2k, const Lists& L,
                              cudaStream_t s) {
  long long warps = (long long)P.Hkv * P.T;
  if (warps == 0) return cudaSuccess;
  long long blocks = (warps + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<true><<<unsigned(blocks), 32 * kTopkWarps, 0, s>>>(P, bmax, q2k, L);
  return cudaGetLastError();
}

}  // namespace msa
