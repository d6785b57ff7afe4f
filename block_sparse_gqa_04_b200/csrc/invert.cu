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
//            128-row tiles each list needs (tile offsets)
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

// One CTA of 1024 threads; each thread owns a contiguous run of lists.
__global__ void __launch_bounds__(1024) scan_kernel(Problem P, Lists L) {
  __shared__ int s_e[1024];
  __shared__ int s_t[1024];
  const long long n = P.nlists;
  const int tid = threadIdx.x;
  const long long per = (n + 1023) / 1024;
  const long long lo = min(n, per * tid), hi = min(n, lo + per);
  int se = 0, st = 0;
  for (long long i = lo; i < hi; ++i) {
    const int c = L.counts[i];
    se += c;
    st += (c + P.qpt - 1) / P.qpt;
  }
  s_e[tid] = se;
  s_t[tid] = st;
  __syncthreads();
  // Hillis-Steele inclusive scan over the 1024 partial sums
  for (int off = 1; off < 1024; off <<= 1) {
    int ae = tid >= off ? s_e[tid - off] : 0;
    int at = tid >= off ? s_t[tid - off] : 0;
    __syncthreads();
    s_e[tid] += ae;
    s_t[tid] += at;
    __syncthreads();
  }
  int ee = s_e[tid] - se, et = s_t[tid] - st;  // exclusive
  for (long long i = lo; i < hi; ++i) {
    const int c = L.counts[i];
    L.list_off[i] = ee;
    L.tile_off[i] = et;
    ee += c;
    et += (c + P.qpt - 1) / P.qpt;
  }
  if (tid == 1023) {
    L.list_off[n] = s_e[1023];
    L.tile_off[n] = s_t[1023];
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

static unsigned grid_for(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  if (b > 148LL * 64) b = 148LL * 64;
  return unsigned(b < 1 ? 1 : b);
}

cudaError_t launch_invert(const Problem& P, const int32_t* q2k, const Lists& L,
                          int32_t* status, cudaStream_t s) {
  const long long n = (long long)P.Hkv * P.T * P.K;
  prep_kernel<<<grid_for(P.nlists, 256), 256, 0, s>>>(P, L);
  count_kernel<<<grid_for(n, 256), 256, 0, s>>>(P, q2k, L, status);
  scan_kernel<<<1, 1024, 0, s>>>(P, L);
  scatter_kernel<<<grid_for(n, 256), 256, 0, s>>>(P, q2k, L);
  return cudaGetLastError();
}

cudaError_t launch_tile_records(const Problem& P, const Lists& L, cudaStream_t s) {
  tile_records_kernel<<<grid_for(max_tiles(P), 256), 256, 0, s>>>(P, L);
  return cudaGetLastError();
}

}  // namespace msa
