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
//   * the softmax warps normalise O by the row sum, stage the bf16 rows in the
//     tile's own Q buffer (free once S is done) and copy them out with
//     coalesced 16-byte stores (each warp its own 32 rows, which are contiguous
//     in the entry-ordered partial states), leaving the TMA unit to the Q
//     gathers; the base-2 log-normaliser goes with them.
// Two softmax warpgroups take alternate tiles, each with its own TMEM buffer
// pair (S|P, O) of 256 columns, so two tiles are in their softmax while the
// tensor cores run the MMAs of their neighbours; a buffer's next S = Q K^T is
// issued as soon as its previous P V has completed, so it overlaps the
// previous tile's epilogue.  Each softmax thread holds its whole S row (and
// later its O row) in registers, so a tile costs one TMEM round trip each.
// Two threads issue the MMAs, one per TMEM buffer (warp 1 the even tiles, warp
// 10 the odd ones), each in a straight line: wait for the tile's descriptor,
// K/V, Q and its buffer's previous P V, issue S, wait for P, issue P V.  (One
// thread polling every barrier of both buffers noticed a ready P up to ~900
// cycles late; two straight-line threads cut the attention by ~4.5 %.)  A
// thread's commits track only its own MMAs, so a K/V buffer is released by the
// last tile of each parity in the list's run (the producer stands in for the
// missing parity of a one-tile run): its empty barrier counts two arrivals.
//
// With fp8 (e4m3) q and k (aiforradalom.online "Elérhetőség": the inference
// kernels come in BF16 and FP8 among others) the score product S = Q K^T runs as
// kind::f8f6f4 MMAs on 128-byte rows (K = 32 per instruction) and P V stays
// bf16.  A query's Q rows are then 2 KB (one 2D box of 16 rows), a Q stage 16 KB,
// so four stages fit, and each stage is released as soon as its S product has
// completed; the output rows are staged in a separate 32 KB area per softmax
// warpgroup instead of the tile's Q stage.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

constexpr int kThreads = 352;                 // warp 0 TMA, warps 1, 10 MMA, warps 2-9 softmax
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
  static constexpr int kQStages = QK8 ? 4 : 3;
  static constexpr int kKBytes = QK8 ? 16384 : kTileBytes; // 128 keys x 128 dims
  static constexpr int kKVBytes = kKBytes + kTileBytes;    // K then V
  static constexpr int kOStageBytes = QK8 ? kTileBytes : 0;  // per warpgroup (else the Q stage)
  static constexpr uint32_t kIdescS =
      QK8 ? tc::idesc_e4m3_f32(128, 128) : tc::idesc_bf16_f32(128, 128, 0, 0);
};

// Tiles are dealt to CTAs block-cyclically in chunks of kChunk consecutive
// tiles: chunk k goes to CTA k % grid.  Consecutive tiles of a list stay on
// one CTA (K/V is loaded once per chunk), while at any moment all CTAs work
// inside the same narrow window of the tile order, i.e. on the same query
// chunk of the same group, whose Q rows then stay resident in L2.
constexpr int kChunk = 8;
constexpr int kDesc = 4;  // tile descriptors in flight

// What the producer warp tells the MMA warp and the softmax warps about a tile.
struct TileDesc {
  int c, e0, n, flags;     // flags: 1 new list, 2 last tile of its list here, 4 kv stage,
                          // 8 last tile of its parity in the list, 16 kv load parity
  int rows[kQPerTile];     // query rows of the gathered queries
};

struct Bars {
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[kMaxQStages], q_empty[kMaxQStages];
  uint64_t s_full[2], p_full[2], o_full[2], buf_empty[2];
  uint64_t d_full[kDesc], d_empty[kDesc];
  TileDesc desc[kDesc];
  uint64_t mma_done;       // the MMA threads' final commits (drain before TMEM is freed)
  uint32_t tmem_base;
  int abort;
};

template <bool QK8>
constexpr size_t smem_bytes() {
  using C = Cfg<QK8>;
  return 1024 + C::kQStages * C::kQStageBytes + 2 * C::kKVBytes + 2 * C::kOStageBytes +
         sizeof(Bars) + 64;
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
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
               Problem P, Lists L,
               float* __restrict__ part_lse, int* __restrict__ status,
               uint8_t* __restrict__ part_o) {
  using C = Cfg<QK8>;
  constexpr int kQStages = C::kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = smem;                                  // [stages]: Q (bf16: then output staging)
  uint8_t* kvbuf = qbuf + kQStages * C::kQStageBytes;    // [2][K | V 32 KB]
  uint8_t* obuf = kvbuf + 2 * C::kKVBytes;               // fp8 q/k: [2][32 KB] output staging
  Bars* bars = reinterpret_cast<Bars*>(obuf + 2 * C::kOStageBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      // bf16: the four warps that stored the tile from it; fp8: the S MMAs' commit
      tc::mbar_init(&bars->q_empty[s], QK8 ? 1 : 4);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->kv_full[s], 1);
      tc::mbar_init(&bars->kv_empty[s], 2);  // both MMA issuers (or one + the producer)
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 4);
      tc::mbar_init(&bars->o_full[s], 1);
      tc::mbar_init(&bars->buf_empty[s], 4);
    }
    for (int d = 0; d < kDesc; ++d) {
      tc::mbar_init(&bars->d_full[d], 1);
      tc::mbar_init(&bars->d_empty[d], 5);  // the tile's MMA thread and its four softmax warps
    }
    tc::mbar_init(&bars->mma_done, 2);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch(&tmap_q);
    tc::tma_prefetch(&tmap_k);
    tc::tma_prefetch(&tmap_v);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int total = __ldg(L.tile_off + P.nlists);
  bool failed = false;

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
  } else if (warp == 1 || warp == 10) {
    // ---------------- MMA issuers: warp 1 the tiles of TMEM buffer 0, warp 10 of buffer 1 ----------------
    const int me = warp == 1 ? 0 : 1;
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
        if (QK8) tc::mma_commit(&bars->q_empty[qs]);  // the Q stage is read
        if (!tc::mbar_spin(&bars->p_full[buf], (ns >> 1) & 1, abort)) { failed = true; break; }
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
  } else if (warp <= 9) {
    // ---------------- softmax + epilogue (two warpgroups) ----------------
    const int wg = (warp - 2) >> 2;          // tiles j with j % 2 == wg, TMEM buffer wg
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
    const uint32_t sbase = tmem + lane_addr + wg * 256;  // S|P at +0, O at +128
    const float sl2 = P.scale * 1.4426950408889634f;
    const int el = row / kGroup, hh = row % kGroup;
    for (int j = wg; tile_of(j) < total; j += 2) {
      const int d = j % kDesc, qs = j % kQStages;
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
      // slots: summing fp32 values saves widening the bf16 ones, -3 % for the
      // kernel), and each pair is rounded once to bf16x2 for the P V product
      const uint64_t sl2x2 = f2(sl2, sl2), nmsx2 = f2(-ms, -ms);
      uint64_t lsum[2] = {0, 0};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pw[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const uint64_t z = fma2((uint64_t(v[q4][x + 1]) << 32) | v[q4][x], sl2x2, nmsx2);
          const float pa = ex2_f32(__uint_as_float(uint32_t(z)));
          const float pb = ex2_f32(__uint_as_float(uint32_t(z >> 32)));
          lsum[(x >> 1) & 1] = add2(lsum[(x >> 1) & 1], f2(pa, pb));
          pw[x >> 1] = pack_bf16(pa, pb);
        }
        tmem_st16(sbase + q4 * 16, pw);  // P columns 16*q4.. (S is all in registers)
      }
      const uint64_t lsx = add2(lsum[0], lsum[1]);
      const float l = __uint_as_float(uint32_t(lsx)) + __uint_as_float(uint32_t(lsx >> 32));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->p_full[wg]);
      if (!warp_wait(&bars->o_full[wg], par, abort)) { failed = true; break; }
      tc::tc_fence_after();
      // Stage the normalised bf16 O row in this tile's Q buffer (bf16 q/k: S is
      // done with it) or in the warpgroup's staging area (fp8 q/k).  Each warp
      // owns 32 consecutive rows (two gathered queries, contiguous in the
      // entry-ordered partial states) and stores them itself.  The staging
      // uses the 128-byte swizzle (16-byte chunk k of a row goes to chunk
      // k ^ (row % 8)), so that the row-per-lane writes and the chunk-per-lane
      // reads both spread over the banks.
      uint8_t* wst = QK8 ? obuf + wg * C::kOStageBytes + quarter * 8192
                         : qbuf + qs * C::kQStageBytes + quarter * 8192;
      const float inv = 1.f / l;
      const uint64_t invx2 = f2(inv, inv);
      uint32_t o[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tc::tmem_ld32(sbase + 128 + q4 * 32, o[q4]);
      tc::tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint8_t* half = wst + (q4 >> 1) * 4096 + lane * 128;
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          const uint32_t* w8 = o[q4] + 8 * k8;
          uint4 u;
          u.x = to_bf16x2(mul2((uint64_t(w8[1]) << 32) | w8[0], invx2));
          u.y = to_bf16x2(mul2((uint64_t(w8[3]) << 32) | w8[2], invx2));
          u.z = to_bf16x2(mul2((uint64_t(w8[5]) << 32) | w8[4], invx2));
          u.w = to_bf16x2(mul2((uint64_t(w8[7]) << 32) | w8[6], invx2));
          const int chunk = (q4 & 1) * 4 + k8;
          *reinterpret_cast<uint4*>(half + ((chunk ^ (lane & 7)) << 4)) = u;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->buf_empty[wg]);
      if (valid) part_lse[(long long)(e0 + el) * kGroup + hh] = ms + __log2f(l);
      // the warp's rows from the staging area to the partial states with
      // coalesced 16-byte stores (two 256-byte rows per instruction), streaming
      // past L2 (the combine reads them once); the load/store units carry them
      // so that the TMA unit is left to the Q gathers
      const int nrows = min(32, n * kGroup - quarter * 32);  // 0, 16 or 32
      uint8_t* gdst = part_o + (size_t(e0) * kGroup + quarter * 32) * 256;
      for (int it = 0; it < nrows / 2; ++it) {
        const int r = 2 * it + (lane >> 4), k = lane & 15;
        const uint4 u = *reinterpret_cast<const uint4*>(wst + (k >> 3) * 4096 + r * 128 +
                                                        (((k & 7) ^ (r & 7)) << 4));
        __stcs(reinterpret_cast<uint4*>(gdst + r * 256 + k * 16), u);
      }
      __syncwarp();
      if (lane == 0) {
        // bf16: the staging area is the tile's Q buffer, free again
        if (!QK8) tc::mbar_arrive(&bars->q_empty[qs]);
        tc::mbar_arrive(&bars->d_empty[d]);
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

bool attn_tc_supported(const Problem& P) {
  return !P.f32 && P.D == 128 && P.G == kGroup && P.Bk == 128 &&
         (long long)P.T * P.Hq < (1LL << 31) && P.kv_rows < (1LL << 31);
}

cudaError_t launch_attn_tc(const Problem& P, const void* q, const void* k, const void* v,
                           const Lists& L, const Partials& part, int32_t* status,
                           cudaStream_t s) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
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
  auto kern = P.qk8 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  const size_t smem = P.qk8 ? smem_bytes<true>() : smem_bytes<false>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  kern<<<sm_count(), kThreads, smem, s>>>(mq, mk, mv, P, L, part.lse2, status,
                                           static_cast<uint8_t*>(part.o));
  return cudaGetLastError();
}

}  // namespace msa
