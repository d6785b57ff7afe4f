// Internal launch interface between the C ABI layer (msa_api.cu) and the
// kernel files.  Not part of the public header.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

// Query rows of one sequence handled as one unit of the block -> query lists.
// The lists are keyed by (sequence, group, query chunk, block) so that the
// queries gathered by one chunk's work stay resident in L2.
constexpr int kQueryChunk = 8192;

// Resolved problem, shared by every launcher.
struct Problem {
  int B, Sq, Skv, Hq, Hkv, D, DI, Bk, K;
  int G;            // query heads per group
  int T;            // B * Sq query rows
  int nblk;         // ceil(Skv / Bk)
  int nqc;          // ceil(Sq / kQueryChunk)
  int qpt;          // gathered queries per 128-row tile = 128 / G
  long long q_pos0;
  float scale;      // main-branch logit scale
  bool f32;         // fp32 tensors (else bf16)
  bool idx8;        // q_idx and k_idx are fp8 e4m3 (bf16 problems)
  bool idx4;        // q_idx and k_idx are NVFP4 codes with ue4m3 scales qsc, ksc
  const uint8_t* qsc;  // NVFP4: [T, Hkv, DI/16] scales of q_idx
  const uint8_t* ksc;  // NVFP4: [kv_rows, DI/16] scales of k_idx
  bool qk8;         // q and k are fp8 e4m3, v bf16 (bf16 problems)
  // KV storage: contiguous per sequence (table == nullptr) or a pool of
  // `pages` pages of Bk tokens named by table[b * nblk + c]
  const int32_t* table;
  int pages;
  long long kv_rows;  // rows of k, v and k_idx in memory: B * Skv or pages * Bk
  long long nlists; // B * Hkv * nqc * nblk
};

// Shape checks of the C ABI: fills *P from *p or returns why it cannot.
msa_status_t resolve_problem(const msa_problem_t* p, Problem* P);
// MSA_OK for cudaSuccess, else MSA_ERR_CUDA with `e` kept for msa_last_cuda_error.
msa_status_t status_of(cudaError_t e);

// Views into the caller's workspace.
struct Lists {
  int32_t* counts;    // [nlists]
  int32_t* cursor;    // [nlists]
  int32_t* list_off;  // [nlists + 1]
  int32_t* tile_off;  // [nlists + 1]
  int32_t* entries;   // [Hkv * T * K] packed (row << 5) | slot, grouped by list
  int32_t* pos;       // [Hkv, T, K] position of (g, row, slot) in entries, or -1
  int32_t* tiles;     // [max_tiles] TileRec, one per 128-row tile (tensor-core path)
  int32_t* seg_sums;  // [2 * ceil(nlists / 2048)] scan scratch
};

// One 128-row tile of gathered queries: everything the KV-outer kernel needs to
// stage it, precomputed so that kernel's producer reads one record per tile.
struct TileRec {
  int c, g, b;        // block, group, sequence
  int e0, n;          // first entry and number of gathered queries (<= 8)
  int tend;           // first tile of the next list
  int lid;            // list id (low 31 bits)
  int pad;
  int rows[8];        // query rows of the gathered queries
};
static_assert(sizeof(TileRec) == 64, "TileRec is 64 bytes");

// Upper bound on the number of 128-row tiles.
inline long long max_tiles(const Problem& P) {
  return (long long)P.Hkv * P.T * P.K / P.qpt + P.nlists + 1;
}

// Partial softmax states, stored in entry order: the G query heads of entry e
// occupy rows e*G .. e*G+G-1, so one tile of gathered queries writes one
// contiguous run.
struct Partials {
  void* o;            // [entries, G, D] bf16 (bf16 problems) or fp32, normalised
  float* lse2;        // [entries, G] base-2 log of the softmax normaliser
};

// --- index branch ---------------------------------------------------------
cudaError_t launch_fill(float* p, size_t n, float value, cudaStream_t s);
// Block maxima with SIMT kernels (any dtype / index_dim).
cudaError_t launch_index_simt(const Problem& P, const void* q_idx, const void* k_idx,
                              float* bmax, cudaStream_t s);
// Block maxima with the tcgen05 / TMA kernel (bf16, index_dim 128).
bool index_tc_supported(const Problem& P);
cudaError_t launch_index_tc(const Problem& P, const void* q_idx, const void* k_idx,
                            float* bmax, int32_t* status, cudaStream_t s);
// Selection fused into the tcgen05 index kernel (no block maxima in HBM): the
// index kernel leaves partial top (k-1) lists per (group, row) in `cand`
// (index_select_cand_bytes), and the merge kernel writes q2k.  For index_tc
// problems with top_k <= 16 and 2 or 4 groups.
bool index_select_fused_supported(const Problem& P);
size_t index_select_cand_bytes(const Problem& P);
cudaError_t launch_index_select(const Problem& P, const void* q_idx, const void* k_idx,
                                void* cand, int32_t* status, cudaStream_t s);
cudaError_t launch_select_merge(const Problem& P, const void* cand, int32_t* q2k,
                                cudaStream_t s);
// Block maxima for a few query rows per sequence (decode): a TMA-fed stream over
// k_idx (bf16, index_dim 128).
bool index_decode_supported(const Problem& P);
cudaError_t launch_index_decode(const Problem& P, const void* q_idx, const void* k_idx,
                                float* bmax, int32_t* status, cudaStream_t s);
cudaError_t launch_topk(const Problem& P, const float* bmax, int32_t* q2k, cudaStream_t s);
// NVFP4 index tensors: block maxima straight from the codes for a few rows per
// sequence (decode), or a bf16 copy of codes x scales for the other index kernels.
bool nvfp4_keys_supported(const Problem& P);
cudaError_t launch_index_nvfp4_keys(const Problem& P, const void* q_codes, const void* k_codes,
                                    float* bmax, cudaStream_t s);
cudaError_t launch_dequant_nvfp4(const void* codes, const uint8_t* scales, void* out_bf16,
                                 long long rows, int di, cudaStream_t s);
// One query row per sequence whose rows all keep top_k blocks (q_pos0 >=
// (top_k-1)*Bk): the top-k kernel also writes the block -> query lists (entries,
// positions, tile records), in the layout launch_lists_direct gives them.
bool topk_writes_lists(const Problem& P);
struct Lists;
cudaError_t launch_topk_lists(const Problem& P, const float* bmax, int32_t* q2k, const Lists& L,
                              cudaStream_t s);

// --- block -> query lists ---------------------------------------------------
cudaError_t launch_invert(const Problem& P, const int32_t* q2k, const Lists& L,
                          int32_t* status, cudaStream_t s);
// Fills L.tiles from the list offsets (one record per tile).
cudaError_t launch_tile_records(const Problem& P, const Lists& L, cudaStream_t s);
// One query row per sequence with the tensor-core attention kernel: entries,
// positions and tile records in one launch (every list has at most one entry).
bool lists_direct(const Problem& P);
cudaError_t launch_lists_direct(const Problem& P, const int32_t* q2k, const Lists& L,
                                int32_t* status, cudaStream_t s);

// --- main branch ------------------------------------------------------------
cudaError_t launch_attn_simt(const Problem& P, const void* q, const void* k, const void* v,
                             const Lists& L, const Partials& part, cudaStream_t s);
bool attn_tc_supported(const Problem& P);
cudaError_t launch_attn_tc(const Problem& P, const void* q, const void* k, const void* v,
                           const Lists& L, const Partials& part, int32_t* status,
                           cudaStream_t s);
cudaError_t launch_combine(const Problem& P, const int32_t* pos, const Partials& part,
                           void* out, float* lse, int32_t* status, cudaStream_t s);

// --- KL-alignment loss of the index branch (training side) --------------------
bool index_kl_supported(const Problem& P);
// kl_rows [Hkv*T] and ds_buf [Hkv*T*K*Bk] are workspace; dk_idx is overwritten.
cudaError_t launch_index_kl(const Problem& P, const void* q, const void* k, const void* q_idx,
                            const void* k_idx, const int32_t* q2k, const Lists& L,
                            float* kl_rows, float* ds_buf, float* loss, float* dq_idx,
                            float* dk_idx, int32_t* status, cudaStream_t s);

// Device status bits (workspace status word): 1 = invalid q2k entry given to
// attend, 2 = a bounded wait inside a tensor-core kernel gave up, 4 = a block
// table page id outside [0, pages).
constexpr int kStatusBadEntry = 1;
constexpr int kStatusBadPage = 4;

// First memory row of block c of sequence b in k, v and k_idx: contiguous
// sequences, or the page the block table names (page 0 for an id outside
// [0, pages), which launch_check_table flags).  Rows of a block are contiguous.
__device__ __forceinline__ long long block_row(const Problem& P, int b, long long c) {
  if (!P.table) return (long long)b * P.Skv + c * P.Bk;
  const int pg = P.table[(long long)b * P.nblk + c];
  return (pg >= 0 && pg < P.pages) ? (long long)pg * P.Bk : 0;
}
// Memory row of token j of sequence b.
__device__ __forceinline__ long long key_row(const Problem& P, int b, long long j) {
  return block_row(P, b, j / P.Bk) + j % P.Bk;
}
// Flags kStatusBadPage for every block table entry outside [0, pages) (paged
// problems only; no launch otherwise).
cudaError_t launch_check_table(const Problem& P, int32_t* status, cudaStream_t s);

// Kernel launches made by each launcher (for msa_launch_count).
constexpr int kLaunchesInvert = 5;

}  // namespace msa
