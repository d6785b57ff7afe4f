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
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM, warps 1 and 10 issue the
// MMAs of the units of accumulator slot 0 and slot 1 (alternate units), warps
// 2-9 load index queries into TMEM and run the epilogue (one query row per
// thread: masked max over the row's 128 columns, one fp32 store per unit).
// The epilogue is two warpgroups, one per accumulator, so that two units drain
// at once while the tensor cores fill the next.  Two issuing threads keep the
// MMA pipe fed: it queues one instruction, and the barrier tests, commits and
// loop work one thread does between its units would otherwise leave it idle
// (one thread: ~950 SM cycles per 512-cycle unit; two: 7 % faster for the GEMM
// and 4 % with the streamed selection at 128K).  A thread's commits track only
// its own MMAs, so the k_idx stage and the query region are released by both
// (their barriers count two arrivals).
//
// Streaming selection (FUSE): instead of writing the block maxima, each
// epilogue thread keeps, for each group its warpgroup drains, the largest
// keys (orderable score, lower id on ties) of the earlier blocks c < floor(t/Bk)
// of its query row, in a descending array of kMaxKeep entries in shared memory
// with its last entry in a register.  A new key enters with a branch-free
// insertion (entry i becomes max(a[i], min(a[i-1], key))), the same
// instructions on every lane, so a warp pays one pass however many of its rows
// take the key ("MiniMax lancerer MSA" (snilld.dk), section "Teknisk forklaring hvorfor
// kompleksiteten skifter": the top-k over raw block scores is where the gain
// can be lost, so the block scores never make an HBM round trip).  A query
// tile's blocks may be split between the contiguous shares of neighbouring
// CTAs; each CTA writes its partial list for the tile to its own slot, and
// select_merge_kernel takes the top (k-1) over the tile's slots, adds the
// local block and writes the ascending selection.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 352;               // TMA, MMA, two epilogue warpgroups, 2nd MMA
constexpr int kMaxGroups = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 256;           // accumulators follow the A region
constexpr int kEpiThreads = 256;            // the two epilogue warpgroups
constexpr int kMaxKeep = 15;                // streaming selection: top_k - 1 <= 15
constexpr size_t kListBytes = size_t(2) * kMaxKeep * kEpiThreads * 8;  // two groups per thread

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
  static constexpr size_t kSmemBytesFused = kSmemBytes + kListBytes;
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

// The CTA whose contiguous share of the pair index contains pair L, for shares
// [total*x/grid, total*(x+1)/grid) (the largest x with total*x/grid <= L).
__host__ __device__ inline int cta_of_pair(long long L, long long total, int grid) {
  return int(((L + 1) * grid + total - 1) / total) - 1;
}

// Position of query tile m in the order of tile_at.
__host__ __device__ inline int order_of_tile(const Problem& P, int m) {
  const int M = mtiles(P);
  return m < (M + 1) / 2 ? 2 * m : 2 * (M - 1 - m) + 1;
}

// Slots of partial selection lists per (group, row): the most CTA shares one
// query tile's pairs can be split into.
inline int select_slots(const Problem& P, long long total, int grid) {
  const long long share = total / grid;  // >= 1: grid <= total
  return int((P.nblk + share - 1) / share) + 1;
}

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t a_full;
  uint64_t a_empty;
  uint64_t mma_done;       // the MMA thread's final commit (drain before TMEM is freed)
  uint32_t tmem_base;
  int abort;
};

template <bool FP8, bool FUSE>
__global__ void __launch_bounds__(kThreads, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, Problem P,
                const uint8_t* __restrict__ q_idx, float* __restrict__ bmax,
                uint64_t* __restrict__ cand, int nslot, int* __restrict__ status,
                long long per_seq) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  using X = Idx<FP8>;
  Bars* bars = reinterpret_cast<Bars*>(smem + kStages * X::kStageBytes);
  // FUSE: kept keys, [group of the warpgroup][entry][epilogue thread]
  uint64_t* keep = reinterpret_cast<uint64_t*>(smem + kStages * X::kStageBytes + 256);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 2);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->acc_full[s], 1);
      tc::mbar_init(&bars->acc_empty[s], 4);
    }
    tc::mbar_init(&bars->a_full, 8);
    tc::mbar_init(&bars->a_empty, 2);
    tc::mbar_init(&bars->mma_done, 2);
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
      tc::ArmedRing armed;
      for (long long L = L0; L < L1; ++L) {
        if (!tc::mbar_wait(&bars->empty[stage], phase ^ 1, abort)) { failed = true; break; }
        tc::mbar_arrive_expect_tx(&bars->full[stage], X::kStageBytes);
        armed.note(stage, phase);
        const int row = int(block_row(P, w.b, w.c));
        uint8_t* dst = stages + stage * X::kStageBytes;
        tc::tma_load_2d(dst, &tmap_k, &bars->full[stage], 0, row);
        if (!FP8) tc::tma_load_2d(dst + X::kHalfBytes, &tmap_k, &bars->full[stage], 64, row);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        w.next(P);
      }
      // every copy issued has landed before the CTA can leave
      if (!armed.drain(bars->full)) failed = true;
    }
  } else if (warp == 1 || warp == 10) {
    // ---------------- MMA issuers: warp 1 the units of slot 0, warp 10 of slot 1 ----------------
    const int me = warp == 1 ? 0 : 1;
    if (lane == 0 && L0 < L1) {
      Walk w;
      w.start(P, L0, per_seq);
      int stage = 0;
      uint32_t phase = 0, a_phase = 0, n = 0;
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
        for (int g = 0; g < P.Hkv; ++g, ++n) {
          const int slot = int(n & 1);
          if (slot != me) continue;
          if (!tc::mbar_spin(&bars->acc_empty[slot], ((n >> 1) & 1) ^ 1, abort)) {
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
        }
        if (failed) break;
        tc::mma_commit(&bars->empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        seg_start = w.next(P);
        if (seg_start || L + 1 == L1) tc::mma_commit(&bars->a_empty);
      }
      // every MMA issued has completed before TMEM is freed
      if (!tc::mma_drain(&bars->mma_done)) failed = true;
    }
  } else if (warp <= 9) {
    // ---------------- index-query loader + epilogue (two warpgroups) ----------------
    const int ewg = (warp - 2) >> 2;        // accumulator slot this warpgroup drains
    const int quarter = warp & 3;           // TMEM lanes this warp may touch
    const int row = quarter * 32 + lane;    // query row inside the tile
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    const int et = threadIdx.x - 64;        // epilogue thread: the keep lists' column
    const int nkeep = P.K - 1;
    // per group of this warpgroup (g = ewg + 2j): the smallest of the kMaxKeep
    // kept keys (0, below every key, while fewer are kept).  The arrays start
    // empty: all zero.
    uint64_t low0 = 0, low1 = 0;
    if (FUSE) {
#pragma unroll
      for (int e = 0; e < 2 * kMaxKeep; ++e) keep[size_t(e) * kEpiThreads + et] = 0;
    }
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
        const long long lim = t - (long long)w.c * 128;   // last visible column (Bk = 128)
        const bool earlier = w.c < int(t >> 7);             // c < floor(t / 128)
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
          if (!FUSE) {
            if (valid) bmax[((long long)g * P.T + r) * P.nblk + w.c] = m;
          } else if (nkeep > 0) {
            // an earlier block of this row (c < floor(t/Bk)) enters the kept
            // keys if it beats the smallest; the insertion runs on every lane
            // of the warp once any lane needs it (0 leaves the array as it is)
            const int j = g >> 1;
            const uint64_t key = (valid && earlier) ? block_key(m, w.c) : 0;
            if (__any_sync(MSA_FULL_MASK, key > (j ? low1 : low0))) {
              uint64_t* kl = keep + size_t(j) * kMaxKeep * kEpiThreads + et;
              uint64_t a[kMaxKeep];
#pragma unroll
              for (int e = 0; e < kMaxKeep; ++e) a[e] = kl[size_t(e) * kEpiThreads];
              uint64_t prev = a[0];
              a[0] = a[0] > key ? a[0] : key;
#pragma unroll
              for (int e = 1; e < kMaxKeep; ++e) {
                const uint64_t up = prev < key ? prev : key;  // min(old a[e-1], key)
                prev = a[e];
                a[e] = a[e] > up ? a[e] : up;
              }
#pragma unroll
              for (int e = 0; e < kMaxKeep; ++e) kl[size_t(e) * kEpiThreads] = a[e];
              if (j) low1 = a[kMaxKeep - 1];
              else low0 = a[kMaxKeep - 1];
            }
          }
        }
        if (FUSE && nkeep > 0 && (w.c + 1 == w.nc || L + 1 == L1)) {
          // end of this CTA's share of the query tile: its partial lists (the
          // nkeep largest kept keys; 0, below every key, where fewer were
          // kept) go to the CTA's slot among the tile's shares, and the arrays
          // start empty again
          const long long T0 = (long long)w.b * per_seq + pairs_before_at(P, w.u, per_seq);
          const int slot = int(blockIdx.x) - cta_of_pair(T0, per_seq * P.B, gridDim.x);
          for (int j = 0; 2 * j + ewg < P.Hkv; ++j) {
            const int g = 2 * j + ewg;
            uint64_t* kl = keep + size_t(j) * kMaxKeep * kEpiThreads + et;
            uint64_t* dst = cand + ((size_t(g) * nslot + slot) * nkeep) * P.T + r;
            for (int e = 0; e < nkeep; ++e)
              if (valid) dst[size_t(e) * P.T] = kl[size_t(e) * kEpiThreads];
#pragma unroll
            for (int e = 0; e < kMaxKeep; ++e) kl[size_t(e) * kEpiThreads] = 0;
          }
          low0 = low1 = 0;
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

// Final selection from the partial lists, one thread per (group, row): the
// top (k-1) keys over the slots of the row's query tile (each slot holds the
// top (k-1) of one CTA's share of the tile's blocks, so their union holds the
// row's top (k-1)), then the local block; ids ascending, -1 padded.
__global__ void __launch_bounds__(256) select_merge_kernel(Problem P,
                                                           const uint64_t* __restrict__ cand,
                                                           int nslot, long long per_seq, int grid,
                                                           int32_t* __restrict__ q2k) {
  const long long n = (long long)P.Hkv * P.T;
  const long long total = per_seq * P.B;
  const int nkeep = P.K - 1;
  for (long long id = blockIdx.x * (long long)blockDim.x + threadIdx.x; id < n;
       id += (long long)gridDim.x * blockDim.x) {
    const int g = int(id / P.T), r = int(id % P.T);
    const int b = r / P.Sq, i = r % P.Sq;
    const long long t = P.q_pos0 + i;
    const int c_t = int(t / P.Bk);
    const int need = min(P.K, c_t + 1) - 1;  // earlier blocks to keep
    // keys kept so far, largest first (0 = none)
    uint64_t top[kMaxKeep];
#pragma unroll
    for (int e = 0; e < kMaxKeep; ++e) top[e] = 0;
    if (need > 0) {
      const int m = i / 128;
      const long long T0 = (long long)b * per_seq + pairs_before_at(P, order_of_tile(P, m), per_seq);
      const int x0 = cta_of_pair(T0, total, grid);
      const int x1 = cta_of_pair(T0 + tile_blocks(P, m) - 1, total, grid);
      for (int sl = 0; sl <= x1 - x0; ++sl) {
        const uint64_t* src = cand + ((size_t(g) * nslot + sl) * nkeep) * P.T + r;
        for (int e = 0; e < nkeep; ++e) {
          uint64_t x = src[size_t(e) * P.T];
          if (x > top[kMaxKeep - 1]) {
            // insertion into the descending list (branch-free exchange chain)
#pragma unroll
            for (int q = 0; q < kMaxKeep; ++q) {
              const uint64_t hi = x > top[q] ? x : top[q];
              x = x > top[q] ? top[q] : x;
              top[q] = hi;
            }
          }
        }
      }
    }
    // the kept block ids (INT_MAX past `need`), sorted ascending by an
    // odd-even transposition network; every kept id is below c_t
    int id16[kMaxKeep];
#pragma unroll
    for (int e = 0; e < kMaxKeep; ++e) id16[e] = e < need ? key_block(top[e]) : INT_MAX;
#pragma unroll
    for (int round = 0; round < kMaxKeep; ++round) {
#pragma unroll
      for (int e = round & 1; e + 1 < kMaxKeep; e += 2) {
        const int lo = min(id16[e], id16[e + 1]), hi = max(id16[e], id16[e + 1]);
        id16[e] = lo;
        id16[e + 1] = hi;
      }
    }
    int32_t* out = q2k + ((long long)g * P.T + r) * P.K;
#pragma unroll
    for (int e = 0; e < kMaxKeep + 1; ++e) {
      if (e >= P.K) break;
      out[e] = e < need ? id16[e] : (e == need ? c_t : -1);
    }
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

// The streamed selection pays off in bf16, where the epilogue's extra work hides
// under the MMAs (index + merge 8.46 ms against 8.3-8.7 ms for the GEMM and the
// top-k kernel at 128K, and 2.4 GB less DRAM traffic).  With fp8 index tensors the
// MMAs take half as long and the epilogue bounds the kernel (7.23 against 6.38 ms),
// so fp8 keeps the block maxima and the top-k kernel.
bool index_select_fused_supported(const Problem& P) {
  return index_tc_supported(P) && !P.idx8 && P.K - 1 <= kMaxKeep && (P.Hkv == 2 || P.Hkv == 4);
}

namespace {

struct Split {
  long long per_seq, total;
  int grid, nslot;
};

Split split_of(const Problem& P) {
  Split sp;
  sp.per_seq = pairs_per_seq(P);
  sp.total = sp.per_seq * P.B;
  sp.grid = int(std::min<long long>(sm_count(), sp.total));
  sp.nslot = select_slots(P, sp.total, sp.grid);
  return sp;
}

template <bool FP8, bool FUSE>
cudaError_t launch_t(const Problem& P, const void* q_idx, const void* k_idx, float* bmax,
                     uint64_t* cand, int32_t* status, cudaStream_t s) {
  using X = Idx<FP8>;
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // k_idx rows of 128 dims, copied as 128-byte-wide boxes of 128 keys (128-byte swizzle)
  CUtensorMap map;
  cuuint64_t dims[2] = {128u, cuuint64_t(P.kv_rows)};
  cuuint64_t strides[1] = {cuuint64_t(X::kRowBytes)};
  cuuint32_t box[2] = {FP8 ? 128u : 64u, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(k_idx), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const Split sp = split_of(P);
  const size_t smem = FUSE ? X::kSmemBytesFused : X::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<FP8, FUSE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  index_tc_kernel<FP8, FUSE><<<sp.grid, kThreads, smem, s>>>(
      map, P, static_cast<const uint8_t*>(q_idx), bmax, cand, sp.nslot, status, sp.per_seq);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_tc(const Problem& P, const void* q_idx, const void* k_idx,
                            float* bmax, int32_t* status, cudaStream_t s) {
  return P.idx8 ? launch_t<true, false>(P, q_idx, k_idx, bmax, nullptr, status, s)
                : launch_t<false, false>(P, q_idx, k_idx, bmax, nullptr, status, s);
}

size_t index_select_cand_bytes(const Problem& P) {
  const Split sp = split_of(P);
  return size_t(P.Hkv) * sp.nslot * std::max(1, P.K - 1) * size_t(P.T) * sizeof(uint64_t);
}

cudaError_t launch_index_select(const Problem& P, const void* q_idx, const void* k_idx,
                                void* cand, int32_t* status, cudaStream_t s) {
  uint64_t* c = static_cast<uint64_t*>(cand);
  return P.idx8 ? launch_t<true, true>(P, q_idx, k_idx, nullptr, c, status, s)
                : launch_t<false, true>(P, q_idx, k_idx, nullptr, c, status, s);
}

cudaError_t launch_select_merge(const Problem& P, const void* cand, int32_t* q2k,
                                cudaStream_t s) {
  const Split sp = split_of(P);
  const long long n = (long long)P.Hkv * P.T;
  const unsigned blocks = unsigned(std::min<long long>((n + 255) / 256, 148LL * 16));
  select_merge_kernel<<<blocks, 256, 0, s>>>(P, static_cast<const uint64_t*>(cand), sp.nslot,
                                              sp.per_seq, sp.grid, q2k);
  return cudaGetLastError();
}

}  // namespace msa
