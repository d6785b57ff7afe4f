// Block -> query lists ("query gather" of the KV-outer loop).
//
// "MiniMax 稀疏注意力" (hyper.ai), sections 摘要 and 引言: the kernels swap the
// FlashAttention loop order so the outer loop runs over KV blocks and gathers
// the queries that selected each block.  A counting sort turns the per-query
// selection q2k[g, r, slot] into one list per (sequence, group, query chunk,
// block), each entry packing (row << 5) | slot:
//   prep     zero the counters
//   count    histogram of list ids (invalid q2k entries flag the status word)
//   scan     exclusive prefix sums of the counts (entry offsets) and of the
//            128-row tiles each list needs (tile offsets), in two passes over
//            segments of lists (segment sums, then offsets)
//   scatter  place each entry at its list offset + an atomic cursor, and record
//            that position per (group, row, slot) for the combine
// The order inside a list is not fixed, which does not change any result: the
// rows of a tile are independent of one another in every later step.
#include "common.cuh"
#include "internal.h"

namespace msa {

__device__ __forceinline__ long long list_id(const Problem& P, int g, int r, int c) {
  const int b = r / P.Sq;
  const int qc = (r % P.Sq) / kQueryChunk;
  return (((long long)b * P.Hkv + g) * P.nqc + qc) * P.nblk + c;
}

// Entry validity shared by count, scatter and combine: -1 is an empty slot,
// anything else must be a block the row can see.
__device__ __forceinline__ int entry_state(const Problem& P, int r, int c) {
  if (c == -1) return 0;
  const long long t = P.q_pos0 + r % P.Sq;
  return (c >= 0 && (long long)c <= t / P.Bk) ? 1 : -1;
}

__global__ void prep_kernel(Problem P, Lists L) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < P.nlists;
       i += (long long)gridDim.x * blockDim.x) {
    L.counts[i] = 0;
    L.cursor[i] = 0;
  }
}

__global__ void count_kernel(Problem P, const int32_t* __restrict__ q2k, Lists L,
                             int32_t* status) {
  const long long n = (long long)P.Hkv * P.T * P.K;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int g = int(e / ((long long)P.T * P.K));
    const int r = int((e / P.K) % P.T);
    const int c = q2k[e];
    const int st = entry_state(P, r, c);
    if (st < 0) atomicOr(status, kStatusBadEntry);
    if (st > 0) atomicAdd(&L.counts[list_id(P, g, r, c)], 1);
  }
}

// Two-kernel exclusive scan of the list counts (entry offsets) and of the
// tiles each list needs (tile offsets).  scan_sums: CTA s sums segment s of
// kScanSeg lists.  scan_apply: CTA s adds the sums of the segments before it
// and scans its own segment.
constexpr int kScanSeg = 2048;  // lists per segment (256 threads x 8)

__device__ __forceinline__ int tiles_of(int count, int qpt) { return (count + qpt - 1) / qpt; }

// block-wide inclusive scan of (a, b) pairs over 256 threads
__device__ __forceinline__ void block_scan2(int& a, int& b, int* sa, int* sb) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(MSA_FULL_MASK, a, o), xb = __shfl_up_sync(MSA_FULL_MASK, b, o);
    if (lane >= o) { a += xa; b += xb; }
  }
  if (lane == 31) { sa[w] = a; sb[w] = b; }
  __syncthreads();
  if (w == 0) {
    int ta = lane < 8 ? sa[lane] : 0, tb = lane < 8 ? sb[lane] : 0;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int xa = __shfl_up_sync(MSA_FULL_MASK, ta, o), xb = __shfl_up_sync(MSA_FULL_MASK, tb, o);
      if (lane >= o) { ta += xa; tb += xb; }
    }
    if (lane < 8) { sa[lane] = ta; sb[lane] = tb; }
  }
  __syncthreads();
  if (w > 0) { a += sa[w - 1]; b += sb[w - 1]; }
}

__global__ void __launch_bounds__(256) scan_sums_kernel(Problem P, Lists L, int2* seg_sums) {
  __shared__ int sa[8], sb[8];
  const long long lo = (long long)blockIdx.x * kScanSeg;
  int e = 0, t = 0;
  for (int k = 0; k < kScanSeg / 256; ++k) {
    const long long i = lo + k * 256 + threadIdx.x;
    if (i < P.nlists) {
      const int c = L.counts[i];
      e += c;
      t += tiles_of(c, P.qpt);
    }
  }
  block_scan2(e, t, sa, sb);
  if (threadIdx.x == 255) seg_sums[blockIdx.x] = make_int2(e, t);
}

__global__ void __launch_bounds__(256) scan_apply_kernel(Problem P, Lists L,
                                                         const int2* __restrict__ seg_sums) {
  __shared__ int sa[8], sb[8];
  __shared__ int base_e, base_t;
  // offsets of this segment: the sums of all segments before it
  int e = 0, t = 0;
  for (int s = threadIdx.x; s < blockIdx.x; s += 256) {
    e += seg_sums[s].x;
    t += seg_sums[s].y;
  }
  block_scan2(e, t, sa, sb);
  if (threadIdx.x == 255) { base_e = e; base_t = t; }
  __syncthreads();
  int run_e = base_e, run_t = base_t;
  const long long lo = (long long)blockIdx.x * kScanSeg;
  for (int k = 0; k < kScanSeg / 256; ++k) {
    const long long i = lo + k * 256 + threadIdx.x;
    const int c = i < P.nlists ? L.counts[i] : 0;
    int ie = c, it = tiles_of(c, P.qpt);
    __syncthreads();  // sa/sb reuse
    block_scan2(ie, it, sa, sb);
    if (i < P.nlists) {
      L.list_off[i] = run_e + ie - c;
      L.tile_off[i] = run_t + it - tiles_of(c, P.qpt);
    }
    // the last thread's inclusive sums advance the running offsets
    __shared__ int tot_e, tot_t;
    if (threadIdx.x == 255) { tot_e = ie; tot_t = it; }
    __syncthreads();
    run_e += tot_e;
    run_t += tot_t;
  }
  if (lo + kScanSeg >= P.nlists && threadIdx.x == 0) {
    L.list_off[P.nlists] = run_e;
    L.tile_off[P.nlists] = run_t;
  }
}

__global__ void scatter_kernel(Problem P, const int32_t* __restrict__ q2k, Lists L) {
  const long long n = (long long)P.Hkv * P.T * P.K;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int g = int(e / ((long long)P.T * P.K));
    const int r = int((e / P.K) % P.T);
    const int slot = int(e % P.K);
    const int c = q2k[e];
    if (entry_state(P, r, c) <= 0) {
      L.pos[e] = -1;
      continue;
    }
    const long long id = list_id(P, g, r, c);
    const int pos = L.list_off[id] + atomicAdd(&L.cursor[id], 1);
    L.entries[pos] = (r << 5) | slot;
    L.pos[e] = pos;
  }
}

// One thread per tile: find its list (binary search over the tile offsets)
// and write the tile's record.
__global__ void tile_records_kernel(Problem P, Lists L) {
  const int total = L.tile_off[P.nlists];
  for (int tile = blockIdx.x * blockDim.x + threadIdx.x; tile < total;
       tile += gridDim.x * blockDim.x) {
    long long lo = 0, hi = P.nlists;  // tile_off[lo] <= tile < tile_off[hi]
    while (hi - lo > 1) {
      const long long mid = (lo + hi) >> 1;
      if (L.tile_off[mid] <= tile) lo = mid; else hi = mid;
    }
    TileRec rec;
    rec.c = int(lo % P.nblk);
    const long long rest = lo / P.nblk;
    rec.g = int((rest / P.nqc) % P.Hkv);
    rec.b = int(rest / ((long long)P.nqc * P.Hkv));
    rec.e0 = L.list_off[lo] + (tile - L.tile_off[lo]) * P.qpt;
    rec.n = min(P.qpt, L.list_off[lo + 1] - rec.e0);
    rec.tend = L.tile_off[lo + 1];
    rec.lid = int(lo & 0x7fffffff);
    rec.pad = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) rec.rows[e] = e < rec.n ? (L.entries[rec.e0 + e] >> 5) : 0;
    reinterpret_cast<TileRec*>(L.tiles)[tile] = rec;
  }
}

// One query row per sequence (decode): every list holds at most one entry, so
// the counting sort degenerates.  One CTA walks the entries in order, keeps
// the valid ones (a block-wide prefix count gives each its position), and
// writes the entry, its position and a one-query tile record directly.  Only
// the tile count at tile_off[nlists] is written of the offsets: the
// tensor-core attention kernel and the combine read nothing else.
constexpr int kDirectThreads = 1024;
constexpr long long kDirectMaxEntries = 1 << 16;

__global__ void __launch_bounds__(kDirectThreads) direct_lists_kernel(Problem P,
                                                                      const int32_t* __restrict__ q2k,
                                                                      Lists L, int32_t* status) {
  __shared__ int wsum[kDirectThreads / 32];
  __shared__ int run;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long n = (long long)P.Hkv * P.T * P.K;
  if (threadIdx.x == 0) run = 0;
  __syncthreads();
  for (long long base = 0; base < n; base += kDirectThreads) {
    const long long e = base + threadIdx.x;
    int g = 0, r = 0, slot = 0, c = -1, st = 0;
    if (e < n) {
      g = int(e / ((long long)P.T * P.K));
      r = int((e / P.K) % P.T);
      slot = int(e % P.K);
      c = q2k[e];
      st = entry_state(P, r, c);
      if (st < 0) atomicOr(status, kStatusBadEntry);
    }
    const int valid = st > 0 ? 1 : 0;
    int incl = valid;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(MSA_FULL_MASK, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
      int x = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(MSA_FULL_MASK, x, o);
        if (lane >= o) x += y;
      }
      wsum[lane] = x;  // inclusive sums over warps
    }
    __syncthreads();
    const int p = run + (w > 0 ? wsum[w - 1] : 0) + incl - valid;
    if (e < n) {
      if (valid) {
        L.entries[p] = (r << 5) | slot;
        L.pos[e] = p;
        TileRec rec;
        rec.c = c;
        rec.g = g;
        rec.b = r / P.Sq;
        rec.e0 = p;
        rec.n = 1;
        rec.tend = p + 1;
        rec.lid = p;
        rec.pad = 0;
        rec.rows[0] = r;
#pragma unroll
        for (int x = 1; x < 8; ++x) rec.rows[x] = 0;
        reinterpret_cast<TileRec*>(L.tiles)[p] = rec;
      } else {
        L.pos[e] = -1;
      }
    }
    __syncthreads();  // everyone has read run and wsum
    if (threadIdx.x == 0) run += wsum[kDirectThreads / 32 - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) L.tile_off[P.nlists] = run;
}

bool lists_direct(const Problem& P) {
  return P.Sq == 1 && attn_tc_supported(P) && (long long)P.Hkv * P.T * P.K <= kDirectMaxEntries;
}

cudaError_t launch_lists_direct(const Problem& P, const int32_t* q2k, const Lists& L,
                                int32_t* status, cudaStream_t s) {
  direct_lists_kernel<<<1, kDirectThreads, 0, s>>>(P, q2k, L, status);
  return cudaGetLastError();
}

static unsigned grid_for(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  if (b > 148LL * 64) b = 148LL * 64;
  return unsigned(b < 1 ? 1 : b);
}

__global__ void check_table_kernel(Problem P, int32_t* status) {
  const long long n = (long long)P.B * P.nblk;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int pg = P.table[i];
    if (pg < 0 || pg >= P.pages) atomicOr(status, kStatusBadPage);
  }
}

cudaError_t launch_check_table(const Problem& P, int32_t* status, cudaStream_t s) {
  if (!P.table) return cudaSuccess;
  check_table_kernel<<<grid_for((long long)P.B * P.nblk, 256), 256, 0, s>>>(P, status);
  return cudaGetLastError();
}

cudaError_t launch_invert(const Problem& P, const int32_t* q2k, const Lists& L,
                          int32_t* status, cudaStream_t s) {
  const long long n = (long long)P.Hkv * P.T * P.K;
  const unsigned segs = unsigned((P.nlists + kScanSeg - 1) / kScanSeg);
  prep_kernel<<<grid_for(P.nlists, 256), 256, 0, s>>>(P, L);
  count_kernel<<<grid_for(n, 256), 256, 0, s>>>(P, q2k, L, status);
  scan_sums_kernel<<<segs, 256, 0, s>>>(P, L, reinterpret_cast<int2*>(L.seg_sums));
  scan_apply_kernel<<<segs, 256, 0, s>>>(P, L, reinterpret_cast<const int2*>(L.seg_sums));
  scatter_kernel<<<grid_for(n, 256), 256, 0, s>>>(P, q2k, L);
  return cudaGetLastError();
}

cudaError_t launch_tile_records(const Problem& P, const Lists& L, cudaStream_t s) {
  tile_records_kernel<<<grid_for(max_tiles(P), 256), 256, 0, s>>>(P, L);
  return cudaGetLastError();
}

}  // namespace msa
