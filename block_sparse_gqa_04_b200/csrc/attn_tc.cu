// Main branch on tcgen05 tensor cores: KV-outer block-sparse attention with
// query gather ("MiniMax 稀疏注意力" (hyper.ai), sections 摘要 and 核心贡献:
// exp-free top-k plus KV-outer sparse attention to keep the tensor cores busy
// under block-granular access; section 引言: the FlashAttention loop order is
// swapped; snilld.dk "Hvad er MSA i praksis": every query head of a group
// attends over the causally visible tokens of the group's selected blocks).
//
// Shapes: bf16 (or fp8 q/k), head_dim 128, 16 query heads per group, block 128.  The work is
// the flat list of 128-row tiles that the block -> query lists define: a tile is
// 8 gathered queries x 16 heads of one (sequence, group, query chunk, block).
// One persistent CTA per SM takes the tiles dealt to it in chunks of kChunk
// consecutive tiles (block-cyclic over the CTAs).  Per tile:
//   * TMA loads the block's K and V (128 keys x 128 dims each, 128-byte swizzle)
//     into one of two buffers, once per list, and gathers the 8 queries' Q rows
//     (16 heads x 128 dims, 4 KB contiguous in memory) with one box per query
//     through a 4D view of Q that lands the two 8-row groups with their two
//     64-dim halves side by side (8-row groups 2 KB apart in the operand),
//     issued by eight lanes at once;
//   * S = Q K^T (both K-major in shared memory) lands in TMEM, one row per lane;
//   * the softmax warps read their row, apply the scale and the causal cut of
//     the local block, and write P (bf16) back over S in TMEM;
//   * O = P V runs with P from TMEM and V as an MN-major shared-memory operand;
//   * the epilogue warps normalise O by the row sum, stage the bf16 rows in a
//     shared-memory area and store them with TMA (each warp its own 32 rows,
//     which are contiguous in the entry-ordered partial states); the softmax
//     warps write the base-2 log-normaliser.
// Two softmax warpgroups take alternate tiles, each with its own TMEM buffer
// pair (S|P, O) of 256 columns, so two tiles are in their softmax while the
// tensor cores run the MMAs of their neighbours.  A fourth warpgroup does the
// epilogue of every tile, so a softmax warpgroup goes from one tile's P
// straight to its next S, which is issued as soon as the previous P V has
// completed.  The warpgroups trade registers (setmaxnreg) so that a softmax
// thread holds its whole S row.  A Q stage is released as soon as its S
// product has completed.
// Two threads issue the MMAs, one per TMEM buffer (warp 1 the even tiles, warp
// 2 the odd ones), each in a straight line: wait for the tile's descriptor,
// K/V, Q and its buffer's previous P V, issue S, wait for P and for the
// epilogue to have read the buffer's previous O, issue P V.  (One thread
// polling every barrier of both buffers noticed a ready P up to ~900 cycles
// late.)  A thread's commits track only its own MMAs, so a K/V buffer is
// released by the last tile of each parity in the list's run (the producer
// stands in for the missing parity of a one-tile run): its empty barrier counts
// two arrivals.
//
// With fp8 (e4m3) q and k (aiforradalom.online "Elérhetőség": the inference
// kernels come in BF16 and FP8 among others) the score product S = Q K^T runs as
// kind::f8f6f4 MMAs on 128-byte rows (K = 32 per instruction) and P V stays
// bf16.  A query's Q rows are then 2 KB (one 2D box of 16 rows), a Q stage 16 KB,
// and four stages fit.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

// warp 0 TMA, warps 1-2 MMA, warp 3 idle, warps 4-11 softmax, warps 12-15 epilogue
constexpr int kThreads = 512;
constexpr int kRows = 128;
constexpr int kTileBytes = kRows * 128 * 2;   // 32 KB: 128 rows x 128 dims of bf16
constexpr int kHalf = kTileBytes / 2;         // one 64-dim half of a bf16 tile
constexpr int kMaxQStages = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescO = tc::idesc_bf16_f32(128, 128, 0, 1);  // V is MN-major
constexpr int kGroup = 16;                    // query heads per group
constexpr int kQPerTile = kRows / kGroup;     // 8 gathered queries

// Buffer plan by the element type of q and k (v is bf16 either way).
template <bool QK8>
struct Cfg {
  static constexpr int kQBox = QK8 ? 2048 : 4096;          // one query's 16 head rows
  static constexpr int kQStageBytes = kQPerTile * kQBox;   // 16 or 32 KB
  static constexpr int kQStages = QK8 ? 4 : 2;
  static constexpr int kKBytes = QK8 ? 16384 : kTileBytes; // 128 keys x 128 dims
  static constexpr int kKVBytes = kKBytes + kTileBytes;    // K then V
  static constexpr uint32_t kIdescS =
      QK8 ? tc::idesc_e4m3_f32(128, 128) : tc::idesc_bf16_f32(128, 128, 0, 0);
};

// Tiles are dealt to CTAs block-cyclically in chunks of kChunk consecutive
// tiles: chunk k goes to CTA k % grid.  Consecutive tiles of a list stay on
// one CTA (K/V is loaded once per chunk), while at any moment all CTAs work
// inside the same narrow window of the tile order, i.e. on the same query
// chunk of the same group, whose Q rows then stay resident in L2.
constexpr int kChunk = 8;
constexpr int kDesc = 6;  // tile descriptors in flight

// What the producer warp tells the MMA threads, the softmax and the epilogue
// warps about a tile.
struct TileDesc {
  int c, e0, n, flags;     // flags: 1 new list, 2 last tile of its list here, 4 kv stage,
                          // 8 last tile of its parity in the list, 16 kv load parity
  int rows[kQPerTile];     // query rows of the gathered queries
};

struct Bars {
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[kMaxQStages], q_empty[kMaxQStages];
  // per TMEM buffer: S computed, P written, O computed, O read by the
  // epilogue, row sums written, row sums read
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2], l_full[2], l_empty[2];
  uint64_t d_full[kDesc], d_empty[kDesc];
  TileDesc desc[kDesc];
  float lsum[2][kRows];    // row sums of P, softmax -> epilogue, per TMEM buffer
  uint64_t mma_done;       // the MMA threads' final commits (drain before TMEM is freed)
  uint32_t tmem_base;
  int abort;
};

template <bool QK8>
constexpr size_t smem_bytes() {
  using C = Cfg<QK8>;
  return 1024 + C::kQStages * C::kQStageBytes + 2 * C::kKVBytes + kTileBytes + sizeof(Bars) + 64;
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448,
              "shared memory of one CTA");

// The j-th tile of this CTA.
__device__ __forceinline__ long long tile_of(int j) {
  return ((long long)(j / kChunk) * gridDim.x + blockIdx.x) * kChunk + j % kChunk;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(MSA_FULL_MASK, tc::mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Maximum of 32 values (four independent chains of three-input maxima).
__device__ __forceinline__ float max32(const uint32_t (&v)[32], float m) {
  float a[4] = {m, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int x = 0; x < 32; x += 2)
    a[(x >> 1) & 3] = max3(a[(x >> 1) & 3], __uint_as_float(v[x]), __uint_as_float(v[x + 1]));
  return fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// Register split between the warpgroups (setmaxnreg acts on a whole
// warpgroup): the CTA is launched with 512 x 128 registers; the producer/MMA
// warpgroup gives 32 of each thread's back, the epilogue 64, and each softmax
// warpgroup takes 48 more (96 + 64 + 2 x 176 = 512 = 4 x 128), so that a
// softmax thread holds its whole S row.  No role spills at these counts.
constexpr int kRegsCtl = 96, kRegsEpi = 64, kRegsSoftmax = 176;
static_assert(kRegsCtl + kRegsEpi + 2 * kRegsSoftmax <= 4 * 128, "register split");
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Two-wide fp32 helpers (sm_100 packed FMA / add / mul on a 64-bit pair).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  return (uint64_t(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// bf16x2 of the two fp32 halves (low half -> low 16 bits), round to nearest even
__device__ __forceinline__ uint32_t to_bf16x2(uint64_t x) {
  return pack_bf16(__uint_as_float(uint32_t(x)), __uint_as_float(uint32_t(x >> 32)));
}
// 2^x in fp32 on the exp2 unit (flushes subnormal results to zero)
__device__ __forceinline__ float ex2_f32(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


template <bool QK8>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
               const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_v,
               const __grid_constant__ CUtensorMap tmap_o32,
               const __grid_constant__ CUtensorMap tmap_o16, Problem P, Lists L,
               float* __restrict__ part_lse, int* __restrict__ status) {
  using C = Cfg<QK8>;
  constexpr int kQStages = C::kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = smem;                                  // [stages]: Q
  uint8_t* kvbuf = qbuf + kQStages * C::kQStageBytes;    // [2][K | V 32 KB]
  uint8_t* obuf = kvbuf + 2 * C::kKVBytes;               // output staging, 32 KB
  Bars* bars = reinterpret_cast<Bars*>(obuf + kTileBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);  // the S MMAs' commit
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 2);  // both MMA issuers (or one + the producer)
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 4);    // the buffer's softmax warps
      tc::mbar_init(&bars->o_full[s], 1);
      tc::mbar_init(&bars->o_empty[s], 4);   // the epilogue warps have read O
      tc::mbar_init(&bars->l_full[s], 4);    // the softmax warps wrote the row sums
      tc::mbar_init(&bars->l_empty[s], 4);   // the epilogue warps read them
    }
    for (int d = 0; d < kDesc; ++d) {
      tc::mbar_init(&bars->d_full[d], 1);
      // the tile's MMA thread, its four softmax warps and the four epilogue warps
      tc::mbar_init(&bars->d_empty[d], 9);
    }
    tc::mbar_init(&bars->mma_done, 2);
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
  bool failed = false;
  static_assert(kThreads == 512, "four warpgroups");

  if (warp < 4) {
   regs_dec<kRegsCtl>();
   if (warp == 0) {
    // ---------------- producer: tile descriptors + TMA ----------------
    // Lane l holds the record of tile jb + l of this CTA (prefetched one batch
    // ahead); lane 0 waits for buffer space and issues the copies tile by tile.
    const TileRec* recs = reinterpret_cast<const TileRec*>(L.tiles);
    // the Q rows of the current query chunk are gathered once per selected
    // block: keep them in L2 ahead of the streaming partial-state writes
    const uint64_t q_policy = tc::policy_evict_last();
    int kv_stage = 0, q_stage = 0;
    uint32_t kv_phase = 0, q_phase = 0;
    int cur_kvs = 0;
    uint32_t cur_kvpar = 0;
    int prev_lid = -1;
    tc::ArmedRing q_armed, kv_armed;  // lane 0: copies issued into each ring
    auto fetch = [&](int j, TileRec& r) -> bool {
      const long long tile = tile_of(j);
      if (tile >= total) return false;
      const uint4* src = reinterpret_cast<const uint4*>(recs + tile);
      uint4* dst = reinterpret_cast<uint4*>(&r);
#pragma unroll
      for (int x = 0; x < 4; ++x) dst[x] = __ldg(src + x);
      return true;
    };
    TileRec cur, nxt;
    bool cur_ok = fetch(lane, cur);
    for (int jb = 0; !failed; jb += 32) {
      if (!__any_sync(MSA_FULL_MASK, cur_ok)) break;
      const bool nxt_ok = fetch(jb + 32 + lane, nxt);  // in flight while this batch is issued
      const int j = jb + lane;
      const long long nt = tile_of(j + 1);
      const int last = cur_ok && !(nt < total && nt < cur.tend);
      // tile j + 1 is the last of the run: j is the last of its parity too
      int next_last = __shfl_down_sync(MSA_FULL_MASK, last, 1);
      {
        const int tend0 = __shfl_sync(MSA_FULL_MASK, nxt.tend, 0);
        const int ok0 = __shfl_sync(MSA_FULL_MASK, nxt_ok ? 1 : 0, 0);
        if (lane == 31) {
          const long long nnt = tile_of(j + 2);
          next_last = ok0 && !(nnt < total && nnt < tend0);
        }
      }
      const int release = cur_ok && (last || (next_last && nt < total && nt < cur.tend));
      int lid_prev = __shfl_up_sync(MSA_FULL_MASK, cur.lid, 1);
      if (lane == 0) lid_prev = prev_lid;
      const int new_list = cur_ok && cur.lid != lid_prev;
      prev_lid = __shfl_sync(MSA_FULL_MASK, cur.lid, 31);
      for (int jj = 0; jj < 32; ++jj) {
        if (!__shfl_sync(MSA_FULL_MASK, cur_ok, jj)) break;
        const int jt = jb + jj;
        const int tc_ = __shfl_sync(MSA_FULL_MASK, cur.c, jj);
        const int tg = __shfl_sync(MSA_FULL_MASK, cur.g, jj);
        const int tb = __shfl_sync(MSA_FULL_MASK, cur.b, jj);
        const int te0 = __shfl_sync(MSA_FULL_MASK, cur.e0, jj);
        const int tn = __shfl_sync(MSA_FULL_MASK, cur.n, jj);
        const int tnew = __shfl_sync(MSA_FULL_MASK, new_list, jj);
        const int tlast = __shfl_sync(MSA_FULL_MASK, last, jj);
        const int trel = __shfl_sync(MSA_FULL_MASK, release, jj);
        int trow[kQPerTile];
#pragma unroll
        for (int e = 0; e < kQPerTile; ++e) trow[e] = __shfl_sync(MSA_FULL_MASK, cur.rows[e], jj);
        bool good = true;
        if (lane == 0) {
          if (tnew) {
            good = tc::mbar_wait(&bars->kv_empty[kv_stage], kv_phase ^ 1, abort);
            if (good) {
              uint64_t* fb = &bars->kv_full[kv_stage];
              tc::mbar_arrive_expect_tx(fb, C::kKVBytes);
              kv_armed.note(kv_stage, kv_phase);
              uint8_t* dst = kvbuf + kv_stage * C::kKVBytes;
              const int key0 = int(block_row(P, tb, tc_));
              tc::tma_load_3d(dst, &tmap_k, fb, 0, tg, key0);  // fp8: all 128 dims
              if (!QK8) tc::tma_load_3d(dst + kHalf, &tmap_k, fb, 64, tg, key0);
              tc::tma_load_3d(dst + C::kKBytes, &tmap_v, fb, 0, tg, key0);
              tc::tma_load_3d(dst + C::kKBytes + kHalf, &tmap_v, fb, 64, tg, key0);
              cur_kvs = kv_stage;
              cur_kvpar = kv_phase;
              // a one-tile run has one issuer: the producer stands in for the other
              if (tlast) tc::mbar_arrive(&bars->kv_empty[kv_stage]);
            }
          }
          good = good && tc::mbar_wait(&bars->q_empty[q_stage], q_phase ^ 1, abort);
          if (good) {
            tc::mbar_arrive_expect_tx(&bars->q_full[q_stage], uint32_t(tn) * C::kQBox);
            q_armed.note(q_stage, q_phase);
          }
        }
        // the Q boxes of the tile, issued together: lane e copies query e
        if (__shfl_sync(MSA_FULL_MASK, good, 0) && lane < tn) {
          const int e = lane;
          int qr = trow[0];
#pragma unroll
          for (int x = 1; x < kQPerTile; ++x) qr = e == x ? trow[x] : qr;
          if (QK8) {
            // one box: the query's 16 heads as 16 rows of 128 fp8 dims (2 KB)
            tc::tma_load_2d_hint(qbuf + q_stage * C::kQStageBytes + e * C::kQBox, &tmap_q,
                                 &bars->q_full[q_stage], 0, qr * P.Hq + tg * kGroup, q_policy);
          } else {
            // one box: the query's 16 heads as two 8-row groups, each group's two
            // 64-dim halves adjacent (1 KB each, 128-byte swizzle)
            tc::tma_load_4d_hint(qbuf + q_stage * C::kQStageBytes + e * C::kQBox, &tmap_q,
                                 &bars->q_full[q_stage], 0, 0, 0,
                                 (qr * P.Hq + tg * kGroup) >> 3, q_policy);
          }
        }
        if (lane == 0) {
          const int d = jt % kDesc;
          good = good && tc::mbar_wait(&bars->d_empty[d], ((jt / kDesc) & 1) ^ 1, abort);
          if (good) {
            TileDesc& D = bars->desc[d];
            D.c = tc_;
            D.e0 = te0;
            D.n = tn;
            D.flags = (tnew ? 1 : 0) | (tlast ? 2 : 0) | (cur_kvs << 2) | (trel ? 8 : 0) |
                      int(cur_kvpar << 4);
#pragma unroll
            for (int e = 0; e < kQPerTile; ++e) D.rows[e] = trow[e];
            tc::mbar_arrive(&bars->d_full[d]);
          }
        }
        if (!__shfl_sync(MSA_FULL_MASK, good, 0)) { failed = true; break; }
        if (tnew) {
          kv_stage ^= 1;
          if (kv_stage == 0) kv_phase ^= 1;
        }
        if (++q_stage == kQStages) { q_stage = 0; q_phase ^= 1; }
      }
      cur = nxt;
      cur_ok = nxt_ok;
    }
    // every copy issued has landed before the CTA can leave (on the abort path
    // too: the copies complete whether or not anyone consumes them)
    if (lane == 0 && !(q_armed.drain(bars->q_full) && kv_armed.drain(bars->kv_full))) failed = true;
    if (lane != 0) failed = false;  // lane 0 speaks for the warp
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: warp 1 the tiles of TMEM buffer 0, warp 2 of buffer 1 ----------------
    const int me = warp - 1;
    if (lane == 0) {
      for (int ns = me; tile_of(ns) < total && !failed; ns += 2) {
        const int d = ns % kDesc, buf = me, qs = ns % kQStages;
        if (!tc::mbar_spin(&bars->d_full[d], (ns / kDesc) & 1, abort)) { failed = true; break; }
        const int flags = bars->desc[d].flags;
        const int kvs = (flags >> 2) & 1;
        if (!tc::mbar_spin(&bars->kv_full[kvs], (flags >> 4) & 1, abort) ||
            !tc::mbar_spin(&bars->q_full[qs], (ns / kQStages) & 1, abort) ||
            !tc::mbar_spin(&bars->o_full[buf], ((ns >> 1) & 1) ^ 1, abort)) {
          failed = true;
          break;
        }
        tc::tc_fence_after();
        const uint32_t qa = tc::smem_addr(qbuf + qs * C::kQStageBytes);
        const uint32_t ka = tc::smem_addr(kvbuf + kvs * C::kKVBytes);
        const uint32_t dt = tmem + buf * 256;
        if (QK8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_ss_f8(dt, tc::sdesc_sw128(qa + kk * 32, 16, 1024),
                          tc::sdesc_sw128(ka + kk * 32, 16, 1024), C::kIdescS, kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * 1024 + (kk & 3) * 32;
            tc::mma_ss(dt, tc::sdesc_sw128(qa + qoff, 16, 2048),
                       tc::sdesc_sw128(ka + off, 16, 1024), C::kIdescS, kk > 0 ? 1u : 0u);
          }
        }
        tc::mma_commit(&bars->s_full[buf]);
        tc::mma_commit(&bars->q_empty[qs]);  // the Q stage is read
        // P is in TMEM, and the epilogue has read this buffer's previous O
        if (!tc::mbar_spin(&bars->p_full[buf], (ns >> 1) & 1, abort) ||
            !tc::mbar_spin(&bars->o_empty[buf], ((ns >> 1) & 1) ^ 1, abort)) {
          failed = true;
          break;
        }
        tc::tc_fence_after();
        const uint32_t va = ka + C::kKBytes;
        const uint32_t o = tmem + buf * 256 + 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(o, tmem + buf * 256 + kk * 8, tc::sdesc_sw128(va + kk * 2048, kHalf, 1024),
                     kIdescO, kk > 0 ? 1u : 0u);
        tc::mma_commit(&bars->o_full[buf]);
        if (flags & 8) tc::mma_commit(&bars->kv_empty[kvs]);
        tc::mbar_arrive(&bars->d_empty[d]);
      }
      // every MMA issued has completed before TMEM is freed
      if (!tc::mma_drain(&bars->mma_done)) failed = true;
    }
   }
  } else if (warp < 12) {
    // ---------------- softmax (two warpgroups) ----------------
    regs_inc<kRegsSoftmax>();
    const int wg = (warp - 4) >> 2;          // tiles j with j % 2 == wg, TMEM buffer wg
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t sbase = tmem + (uint32_t(quarter * 32) << 16) + wg * 256;  // S|P
    const float sl2 = P.scale * 1.4426950408889634f;
    const int el = row / kGroup, hh = row % kGroup;
    for (int j = wg; tile_of(j) < total; j += 2) {
      const int d = j % kDesc;
      const uint32_t par = (j >> 1) & 1;
      if (!warp_wait(&bars->d_full[d], (j / kDesc) & 1, abort)) { failed = true; break; }
      const TileDesc& D = bars->desc[d];
      const int c = D.c, e0 = D.e0, n = D.n;
      const bool valid = el < n;
      const long long t = P.q_pos0 + (valid ? D.rows[el] : 0) % P.Sq;
      // last visible column of this row in block c (127 = the whole block)
      const int lim = valid ? int(min(127LL, t - (long long)c * P.Bk)) : 127;
      const bool full = __all_sync(MSA_FULL_MASK, lim >= 127);
      if (!warp_wait(&bars->s_full[wg], par, abort)) { failed = true; break; }
      tc::tc_fence_after();
      // the whole S row in registers: four loads, one wait
      uint32_t v[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tc::tmem_ld32(sbase + q4 * 32, v[q4]);
      tc::tmem_ld_wait();
      if (!full) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (q4 * 32 + x > lim) v[q4][x] = __float_as_uint(-INFINITY);
      }
      float m = max32(v[0], -INFINITY);
      m = fmaxf(fmaxf(m, max32(v[1], -INFINITY)), fmaxf(max32(v[2], -INFINITY),
                                                       max32(v[3], -INFINITY)));
      const float ms = m * sl2;
      // P = 2^(S*scale*log2e - max), written over S as bf16, and its sum in
      // fp32, two columns at a time: the scaled logits come from packed fp32x2
      // FMAs, the exponentials from the fp32 exp2 (the exp2 unit takes the same
      // time per value in fp32 as in bf16x2, and this loop is bound by issue
      // slots: summing fp32 values saves widening the bf16 ones), and each pair
      // is rounded once to bf16x2 for the P V product
      const uint64_t sl2x2 = f2(sl2, sl2), nmsx2 = f2(-ms, -ms);
      uint64_t lsum[2] = {0, 0};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
        for (int x8 = 0; x8 < 2; ++x8) {
          uint32_t pw[8];
#pragma unroll
          for (int x = 0; x < 16; x += 2) {
            const uint32_t* s2 = v[q4] + x8 * 16 + x;
            const uint64_t z = fma2((uint64_t(s2[1]) << 32) | s2[0], sl2x2, nmsx2);
            const float pa = ex2_f32(__uint_as_float(uint32_t(z)));
            const float pb = ex2_f32(__uint_as_float(uint32_t(z >> 32)));
            lsum[(x >> 1) & 1] = add2(lsum[(x >> 1) & 1], f2(pa, pb));
            pw[x >> 1] = pack_bf16(pa, pb);
          }
          tmem_st8(sbase + q4 * 16 + x8 * 8, pw);  // P columns 16*q4 + 8*x8 ..
        }
      }
      const uint64_t lsx = add2(lsum[0], lsum[1]);
      const float l = __uint_as_float(uint32_t(lsx)) + __uint_as_float(uint32_t(lsx >> 32));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->p_full[wg]);
      // the row sum to the epilogue (its slot is free once the epilogue has
      // read the buffer's previous one)
      if (!warp_wait(&bars->l_empty[wg], par ^ 1, abort)) { failed = true; break; }
      bars->lsum[wg][row] = l;
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&bars->l_full[wg]);
        tc::mbar_arrive(&bars->d_empty[d]);
      }
      if (valid) part_lse[(long long)(e0 + el) * kGroup + hh] = ms + __log2f(l);
    }
  } else {
    // ---------------- epilogue: every tile in order ----------------
    regs_dec<kRegsEpi>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    // Each warp owns 32 consecutive rows (two gathered queries, contiguous in
    // the entry-ordered partial states) and stores them itself with TMA.  The
    // staging uses the 128-byte swizzle (16-byte chunk k of a row goes to chunk
    // k ^ (row % 8)), which the TMA store undoes.
    uint8_t* wst = obuf + quarter * 8192;
    // partial states are read once, by the combine: first out of L2
    const uint64_t o_policy = tc::policy_evict_first();
    for (int j = 0; tile_of(j) < total; ++j) {
      const int b = j & 1, d = j % kDesc;
      const uint32_t par = (j >> 1) & 1;
      if (!warp_wait(&bars->d_full[d], (j / kDesc) & 1, abort) ||
          !warp_wait(&bars->l_full[b], par, abort)) {
        failed = true;
        break;
      }
      const int e0 = bars->desc[d].e0, n = bars->desc[d].n;
      const float inv = 1.f / bars->lsum[b][row];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->l_empty[b]);
      if (!warp_wait(&bars->o_full[b], par, abort)) { failed = true; break; }
      tc::tc_fence_after();
      // the warp's previous stores have read the staging area
      if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      __syncwarp();
      const uint64_t invx2 = f2(inv, inv);
      const uint32_t obase = tmem + lane_addr + b * 256 + 128;
      // O in four 32-column pieces (the buffer's next P V needs O only after
      // that buffer's next S and softmax, so the round trips cost nothing)
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[32];
        tc::tmem_ld32(obase + q4 * 32, o);
        tc::tmem_ld_wait();
        if (q4 == 3) {
          // all of O has been read: the buffer's next P V may overwrite it
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->o_empty[b]);
        }
        // columns 32*q4 ..: 64-dim half q4 / 2, 16-byte chunks 4*(q4 % 2) ..
        uint8_t* hp = wst + (q4 >> 1) * 4096 + lane * 128;
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          const uint32_t* w8 = o + 8 * k8;
          uint4 u;
          u.x = to_bf16x2(mul2((uint64_t(w8[1]) << 32) | w8[0], invx2));
          u.y = to_bf16x2(mul2((uint64_t(w8[3]) << 32) | w8[2], invx2));
          u.z = to_bf16x2(mul2((uint64_t(w8[5]) << 32) | w8[4], invx2));
          u.w = to_bf16x2(mul2((uint64_t(w8[7]) << 32) | w8[6], invx2));
          const int chunk = (q4 & 1) * 4 + k8;
          *reinterpret_cast<uint4*>(hp + ((chunk ^ (lane & 7)) << 4)) = u;
        }
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int nrows = min(32, n * kGroup - quarter * 32);  // 0, 16 or 32
        if (nrows > 0) {
          const CUtensorMap* map = nrows == 32 ? &tmap_o32 : &tmap_o16;
          const int grow = e0 * kGroup + quarter * 32;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tc::tma_store_2d_hint(map, wst + h * 4096, 64 * h, grow, o_policy);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        tc::mbar_arrive(&bars->d_empty[d]);
      }
    }
    // every store has completed before the CTA exits
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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
         (long long)P.T * P.Hq < (1LL << 31) && P.kv_rows < (1LL << 31);
}

cudaError_t launch_attn_tc(const Problem& P, const void* q, const void* k, const void* v,
                           const Lists& L, const Partials& part, int32_t* status,
                           cudaStream_t s) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mo32, mo16;
  const CUtensorMapDataType qk_type =
      P.qk8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t qk_row = P.qk8 ? 128 : 256;  // bytes of one 128-dim row of q or k
  if (P.qk8) {
    // Q rows (token, head) of 128 fp8 dims: one 16-row box per gathered query
    cuuint64_t dims[2] = {128, cuuint64_t(P.T) * P.Hq};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, kGroup};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&mq, qk_type, 2, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // Q rows (token, head) of 128 dims viewed as (64 dims, 8 rows, 2 halves, row groups)
    cuuint64_t dims[4] = {64, 8, 2, cuuint64_t(P.T) * P.Hq / 8};
    cuuint64_t strides[3] = {128 * 2, 64 * 2, 8 * 128 * 2};
    cuuint32_t box[4] = {64, 8, 2, kGroup / 8};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&mq, qk_type, 4, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // K (fp8: one 128-byte box row per key) and V (bf16: two 64-dim halves)
    cuuint64_t dims[3] = {128, cuuint64_t(P.Hkv), cuuint64_t(P.kv_rows)};
    cuuint64_t kstr[2] = {qk_row, cuuint64_t(P.Hkv) * qk_row};
    cuuint64_t vstr[2] = {128 * 2, cuuint64_t(P.Hkv) * 128 * 2};
    cuuint32_t kbox[3] = {P.qk8 ? 128u : 64u, 1, 128};
    cuuint32_t vbox[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&mk, qk_type, 3, const_cast<void*>(k), dims, kstr, kbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v), dims, vstr, vbox,
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
  auto kern = P.qk8 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  const size_t smem = P.qk8 ? smem_bytes<true>() : smem_bytes<false>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  // The warpgroups' setmaxnreg split draws on the registers the CTA is
  // launched with; a build that gave the kernel fewer than the split adds up
  // to would leave the softmax warpgroups waiting for registers forever, so
  // such a build is refused here.
  static int regs[2] = {0, 0};  // per instantiation, looked up once
  int& nregs = regs[P.qk8 ? 1 : 0];
  if (nregs == 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    nregs = fa.numRegs;
  }
  if (nregs * 4 < kRegsCtl + kRegsEpi + 2 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
  kern<<<sm_count(), kThreads, smem, s>>>(mq, mk, mv, mo32, mo16, P, L, part.lse2, status);
  return cudaGetLastError();
}

}  // namespace msa
