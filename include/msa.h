/*
 * msa.h - C ABI of libmsa, the B200 (sm_100a) MiniMax Sparse Attention (MSA)
 * forward path.
 *
 * MSA splits attention into two branches.  The index branch scores every
 * causally visible key token with one index-query head per GQA group against a
 * single shared index-key head, max-pools the scores to blocks of 128 tokens
 * and keeps, per (query, GQA group), the top-k blocks with the query's own
 * block always among them.  The main branch then runs exact softmax attention
 * of every query head of the group over the causally visible tokens of those
 * blocks only.  Sources: "MiniMax 稀疏注意力" (hyper.ai page of paper
 * 2606.13392), section 摘要; "MiniMax lancerer MSA" (snilld.dk), section
 * "Hvad er MSA i praksis"; "Substantial numerical differences with Minimax MSA
 * attention vs Minimax's Reference", sections 原因分析 and 解决步骤.
 *
 * Conventions for every entry point
 *  - Tensors are dense, row-major, on the current CUDA device, and start on a
 *    16-byte boundary:
 *        q, out   [batch, q_len, num_q_heads, head_dim]
 *        k, v     [batch, kv_len, num_kv_heads, head_dim]
 *        q_idx    [batch, q_len, num_kv_heads, index_dim]
 *        k_idx    [batch, kv_len, index_dim]       (one shared index-key head)
 *    (with a paged KV cache, num_pages > 0, k, v and k_idx are page pools:
 *        k, v     [num_pages, 128, num_kv_heads, head_dim]
 *        k_idx    [num_pages, 128, index_dim]
 *     and block_table [batch, ceil(kv_len/128)] names each block's page)
 *        q2k      [num_kv_heads, batch*q_len, top_k]  int32
 *        lse      [batch, q_len, num_q_heads]      float32
 *        block_scores [num_kv_heads, batch*q_len, nblk] float32,
 *                 nblk = ceil(kv_len / block_size)
 *    The token-major layout and the q2k list layout are the ones the fix in
 *    "Substantial numerical differences ...", section 解决步骤, hands to the
 *    kernel path (q2k[num_kv_heads, bsz*q_len, topk]).
 *  - Query row r = b*q_len + i sits at absolute position t = q_pos0 + i of
 *    sequence b and sees keys 0..t of that sequence.  Query head h belongs to
 *    group g = h / (num_q_heads / num_kv_heads) (contiguous groups, as the
 *    repeat_interleave expansion in section 解决步骤 implies).
 *  - The caller owns every buffer, the workspace included.  The library
 *    allocates no memory, never synchronises the stream, and returns once the
 *    work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Argument errors are returned synchronously, before any launch, and leave
 *    every output untouched.  A failed launch returns MSA_ERR_CUDA.  Problems
 *    found on the device (a q2k entry outside [-1, floor(t/block_size)] given
 *    to msa_attend: bit 1; a block_table page id outside [0, num_pages): bit 4)
 *    are recorded in the workspace status word, read with msa_device_status();
 *    such entries are skipped, such pages read as page 0.
 *  - q_len == 0 is a valid empty problem: the call returns MSA_OK without
 *    looking at the pointers or launching anything.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, bad size or shape */
  MSA_ERR_UNSUPPORTED = 2,   /* valid shape outside what the kernels cover    */
  MSA_ERR_WORKSPACE = 3,     /* ws_bytes smaller than msa_workspace_size()    */
  MSA_ERR_CUDA = 4,          /* a CUDA call or launch failed                  */
  MSA_ERR_DEVICE = 5,        /* the device recorded an invalid q2k entry      */
  MSA_ERR_TOO_LARGE = 6      /* problem exceeds msa_select_static's scratch   */
} msa_status_t;

/* MSA_FP8_E4M3 is an index_dtype or qk_dtype only: fp8 e4m3 index queries and
 * keys, or main-branch queries and keys, of a bf16 problem ("MiniMax új
 * eljárása ..." (aiforradalom.online), section "Elérhetőség": the MSA inference
 * kernels come in BF16, FP8, NVFP4 and FP4).  MSA_NVFP4 is an index_dtype only:
 * NVFP4 index queries and keys of a bf16 problem, e2m1 codes two per byte
 * (element 2i in the low nibble) with one unsigned e4m3 scale byte per 16
 * consecutive elements of index_dim (q_idx_scale, k_idx_scale); a value is
 * e2m1(code) x scale, and scale bytes 0x7f and above are invalid. */
typedef enum { MSA_BF16 = 0, MSA_F32 = 1, MSA_FP8_E4M3 = 2, MSA_NVFP4 = 3 } msa_dtype_t;

typedef enum {
  MSA_OP_SELECT = 0,
  MSA_OP_ATTEND = 1,
  MSA_OP_FORWARD = 2,
  MSA_OP_INDEX_KL = 3 /* msa_index_kl (training side) */
} msa_op_t;

/* One MSA problem.  Supported: block_size 128; top_k 1..32; head_dim 64 or
 * 128; index_dim 32, 64 or 128; num_q_heads a multiple of num_kv_heads with at
 * most 128 query heads per group, dividing 128; q_pos0 + q_len <= kv_len;
 * batch*q_len*32 < 2^31. */
typedef struct {
  int32_t batch;          /* sequences                                         */
  int32_t q_len;          /* query rows per sequence                           */
  int32_t kv_len;         /* key tokens per sequence                           */
  int32_t num_q_heads;
  int32_t num_kv_heads;   /* GQA groups = index-query heads                    */
  int32_t head_dim;       /* D of q, k, v                                      */
  int32_t index_dim;      /* d of q_idx, k_idx                                 */
  int32_t block_size;     /* Bk, tokens per KV block: 128 (every kernel), or 64
                             and 32 (CUDA-core kernels only)                   */
  int32_t top_k;          /* blocks kept per (query, group), local one included */
  int32_t dtype;          /* msa_dtype_t of q, k, v, q_idx, k_idx and out (see
                             index_dtype and qk_dtype for fp8 inputs)          */
  int64_t q_pos0;         /* absolute position of query row 0 of every sequence */
  float softmax_scale;    /* main-branch logit scale; 0 selects 1/sqrt(head_dim) */
  int32_t index_dtype;    /* 0: q_idx and k_idx have `dtype`; MSA_FP8_E4M3: they are
                             fp8 e4m3; MSA_NVFP4: they are NVFP4 codes
                             [.., index_dim/2] uint8 with the scales below (both
                             bf16 problems only); other values are invalid       */
  int32_t qk_dtype;       /* 0: q and k have `dtype`; MSA_FP8_E4M3: q and k are fp8
                             e4m3 and the main-branch scores q . k are formed from
                             them (bf16 problems; v, out and the partial states stay
                             bf16); other values are invalid                      */
  int32_t num_pages;      /* 0: k, v and k_idx are contiguous per sequence (the
                             layouts below).  > 0: paged KV cache: k and v are
                             [num_pages, 128, num_kv_heads, head_dim] and k_idx
                             [num_pages, 128, index_dim], and block_table maps
                             block c of sequence b (tokens c*128 .. c*128+127) to
                             page block_table[b * ceil(kv_len/128) + c]; pages may
                             be shared between sequences.  Rows of a sequence's last
                             page beyond kv_len are read and weighted by zero, so
                             they must hold finite values.  Requires block_size 128 */
  const int32_t* block_table; /* device, [batch, ceil(kv_len/128)] int32 page ids in
                             [0, num_pages) (num_pages > 0), else ignored; an id
                             outside that range sets status bit 4 and reads page 0 */
  const uint8_t* q_idx_scale; /* device, index_dtype MSA_NVFP4 only (else ignored):
                             ue4m3 scales of q_idx, [batch, q_len, num_kv_heads,
                             index_dim/16]                                        */
  const uint8_t* k_idx_scale; /* device, MSA_NVFP4 only: scales of k_idx, [batch,
                             kv_len, index_dim/16] (paged: [num_pages, 128,
                             index_dim/16]); both must be non-NULL for MSA_NVFP4  */
} msa_problem_t;

/* Bytes of workspace that `op` needs for problem `p` (0 if p is invalid).
 * The workspace must start on a 256-byte boundary. */
size_t msa_workspace_size(const msa_problem_t* p, int32_t op);

/* Index branch.  Computes, for every row r and group g, the block maxima of
 * the raw index scores q_idx[r,g,:] . k_idx[b,j,:] over the visible tokens
 * j <= t of each block ("Substantial numerical differences ...", section
 * 原因分析: amax over the block; snilld.dk "Hvad er MSA i praksis": one
 * index-query head per group, one shared index-key head), then writes q2k[g, r]
 * = the local block floor(t/Bk) plus the min(top_k, visible blocks) - 1
 * highest-scoring earlier blocks, ranked on raw scores without exponentials
 * (snilld.dk, "Teknisk forklaring hvorfor kompleksiteten skifter"), ties to the
 * lower block id, ids ascending, -1 padded.
 * block_scores_opt: optional; if not NULL receives the block maxima, with
 * -inf for every block that row r cannot see. */
msa_status_t msa_select(const msa_problem_t* p, const void* q_idx, const void* k_idx,
                        int32_t* q2k, float* block_scores_opt,
                        void* ws, size_t ws_bytes, void* stream);

/* Main branch over a given selection q2k (entries -1 are skipped; others must
 * be visible blocks, 0 <= c <= floor(t/Bk)).  Every query head of group g
 * attends over the visible tokens of the blocks q2k[g, r, :] with softmax
 * scale p->softmax_scale (snilld.dk "Hvad er MSA i praksis": scaled
 * dot-product softmax over exactly those tokens).  Writes out (`dtype`) and,
 * if lse_opt is not NULL, the natural-log softmax normaliser per (row, head);
 * a row with no valid block gets zeros and -inf. */
msa_status_t msa_attend(const msa_problem_t* p, const void* q, const void* k, const void* v,
                        const int32_t* q2k, void* out, float* lse_opt,
                        void* ws, size_t ws_bytes, void* stream);

/* msa_select followed by msa_attend ("MiniMax 稀疏注意力", section 摘要).
 * q2k_opt: optional; if not NULL receives the selection, else the selection
 * lives in the workspace. */
msa_status_t msa_forward(const msa_problem_t* p, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, void* out, float* lse_opt,
                         int32_t* q2k_opt, void* ws, size_t ws_bytes, void* stream);

/* Packed variable-length batch ("Substantial numerical differences with Minimax
 * MSA attention vs Minimax's Reference", section 原因分析: the selection has the
 * packed shape [total_qo_len, heads, topk], the query rows of all sequences
 * concatenated).  Sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 * and key rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 of the packed, token-major
 *   q, out [total_q, num_q_heads, head_dim]   q_idx [total_q, num_kv_heads, index_dim]
 *   k, v   [total_k, num_kv_heads, head_dim]  k_idx [total_k, index_dim]
 *   lse_opt [total_q, num_q_heads] fp32       q2k_opt [num_kv_heads, total_q, top_k] int32
 * Its n_q = cu_seqlens_q[b+1] - cu_seqlens_q[b] query rows are its last n_q tokens
 * (positions n_k - n_q + i, n_k = cu_seqlens_k[b+1] - cu_seqlens_k[b]), as in
 * chunked prefill and decode; 0 <= n_q <= n_k; sequences never see one another.
 * cu_seqlens_q and cu_seqlens_k are HOST arrays of batch + 1 int32 prefix sums
 * starting at 0 (the call reads them before it returns).  p: batch = number of
 * sequences; q_len, kv_len and q_pos0 are ignored; num_pages must be 0
 * (MSA_ERR_UNSUPPORTED otherwise); the other fields and every shape rule as in
 * msa_forward, applied to each sequence.  lse_opt requires num_q_heads % 4 == 0.
 * Consecutive sequences with equal (n_q, n_k) form one batched problem and run
 * as one set of kernel launches; the runs execute one after another on `stream`
 * in the same workspace (msa_varlen_workspace_size bytes: that of the largest
 * run); sequences without query rows cost nothing.  Returns before any launch
 * for bad lengths (a decreasing prefix sum, n_q > n_k), null or misaligned
 * pointers, or a short workspace.  Stage events (msa_set_stage_events) cover the
 * first run. */
msa_status_t msa_forward_varlen(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, const void* q, const void* k,
                                const void* v, const void* q_idx, const void* k_idx, void* out,
                                float* lse_opt, int32_t* q2k_opt, void* ws, size_t ws_bytes,
                                void* stream);

/* Workspace bytes of msa_forward_varlen for these lengths (0 if invalid). */
size_t msa_varlen_workspace_size(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                 const int32_t* cu_seqlens_k);

/* Kernel launches one msa_forward_varlen call makes for these lengths (the sum
 * over its runs of msa_launch_count(run, MSA_OP_FORWARD)); 0 if invalid. */
int32_t msa_varlen_launch_count(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k);

/* msa_select without a workspace: the same index branch and selection,
 * writing the same q2k, with its scratch in a fixed 256-byte-aligned device
 * buffer inside this library (status word + block maxima), so the call
 * allocates no memory at all and takes no workspace.  The pages have no
 * counterpart of this entry point; it is for callers that cannot hand the
 * library device memory: a host runtime that has reserved the whole device up
 * front (a KV-cache pool, say) and has no allocator left to lend, or a C caller
 * without a device allocator.
 *  - Limit: the block maxima, num_kv_heads * batch * q_len * nblk * 4 bytes,
 *    must fit in 4 MiB (e.g. 32 decode rows at 1M tokens with 4 groups);
 *    larger problems return MSA_ERR_TOO_LARGE before anything is launched.
 *  - Setup: the first call on each device (with that device current) looks up
 *    the buffer's address with cudaGetSymbolAddress, which may load the
 *    library's device code; make that first call before any stream capture.
 *  - The buffer is shared by every call on a device: calls whose work overlaps
 *    on the GPU (other streams, other threads) race on it and must be
 *    serialised by the caller.
 *  - Each call clears the status word first (the only scratch that must start
 *    at zero).  device_status_opt: optional device int32; if not NULL it
 *    receives, in stream order, the call's status word, a bitmask as in
 *    msa_device_status (0 = fine).
 *  - The buffer's address is cached per device index for the life of the
 *    process: it assumes one CUDA context per device.  After cudaDeviceReset
 *    (or anything else that tears down and recreates the device's primary
 *    context) the cached address is stale; do not call this entry point
 *    again in that process.
 * Other arguments and errors as msa_select. */
msa_status_t msa_select_static(const msa_problem_t* p, const void* q_idx, const void* k_idx,
                               int32_t* q2k, int32_t* device_status_opt, void* stream);

/* KL-alignment loss of the index branch and its gradients (training side).
 * snilld.dk "Træning og stabilisering": Top-k is not differentiable, so an
 * extra KL-alignment loss trains the index projections, the index branch
 * matching the main branch, whose group-averaged distribution over the selected
 * tokens is the teacher, with gradient detach.  For every row r and group g,
 * over the causally visible tokens J of the blocks q2k[g, r, :] (as msa_select
 * writes them):
 *   p_I = softmax_j(q_idx[r,g] . k_idx[j])                       (raw scores)
 *   p_T = mean over the group's heads h of softmax_j(scale * q[r,h] . k[j,g])
 *   kl  = sum_j p_T[j] (ln p_T[j] - ln p_I[j])
 * Writes *loss (device, one float) = the mean of kl over the batch*q_len*
 * num_kv_heads pairs, and the gradients of that mean with respect to q_idx
 * (dq_idx, fp32, [batch, q_len, num_kv_heads, index_dim]) and k_idx (dk_idx,
 * fp32, [batch, kv_len, index_dim], overwritten) with q, k and q2k held constant
 * (no gradient reaches q or k).  q, k, q_idx, k_idx take the problem's dtypes
 * (qk_dtype, index_dtype).  Workspace: msa_workspace_size(p, MSA_OP_INDEX_KL).
 * q2k entries outside the row's visible blocks are skipped and flag the status
 * word (1), as in msa_attend.  Runs on CUDA cores; MSA_ERR_UNSUPPORTED for block
 * sizes other than 128 and when the per-(row, group) working set (group heads x
 * head_dim + 2 x top_k x 128 floats) exceeds 200 KB of shared memory.  Other
 * errors as msa_attend. */
msa_status_t msa_index_kl(const msa_problem_t* p, const void* q, const void* k,
                          const void* q_idx, const void* k_idx, const int32_t* q2k,
                          float* loss, float* dq_idx, float* dk_idx, void* ws, size_t ws_bytes,
                          void* stream);

/* Reads the workspace status word written by the last call that used `ws`:
 * waits for `stream`, stores the device code in *code and returns MSA_OK if it
 * is 0, else MSA_ERR_DEVICE.  The code is a bitmask (an OR of every problem the
 * call's kernels met): 1 = a q2k entry outside the row's visible blocks
 * (skipped), 2 = a bounded wait inside a tensor-core kernel gave up (the
 * kernel's output is incomplete), 4 = a block_table page id outside
 * [0, num_pages) (read as page 0).  This call synchronises. */
msa_status_t msa_device_status(const void* ws, int32_t* code, void* stream);

/* Stage timing (a measurement aid, not part of the method).  When `events` is
 * not NULL, every later call of msa_select, msa_attend or msa_forward records
 * events[i] (cudaEvent_t values) on its stream right after its i-th stage, for
 * i < n, so the caller can time each kernel with cudaEventElapsedTime against
 * an event recorded before the call; each call numbers its stages from 0, so
 * the same events are recorded again by the next call.  Stages of msa_forward
 * in order: 0 index scores, 1 top-k select, 2 block -> query lists (a few small
 * kernels), 3 KV-outer attention, 4 combine; msa_select records its stages 0-1
 * and msa_attend its stages 0-2 (lists, attention, combine).  The setting is
 * process-wide and not thread-safe; NULL turns it off.  Returns the number of
 * stages of msa_forward. */
int32_t msa_set_stage_events(void* const* events, int32_t n);

/* Number of kernel launches one call of `op` makes for problem `p` (without
 * block_scores_opt, which adds one fill launch). */
int32_t msa_launch_count(const msa_problem_t* p, int32_t op);

/* Which kernel family a call of `op` runs for `p`: a static string naming the
 * index-branch and main-branch kernels ("tc" = tcgen05/TMA path, "simt"). */
const char* msa_kernel_path(const msa_problem_t* p, int32_t op);

/* Self-test of the bounded waits (a diagnostic, not part of the method).
 * Every wait of the tensor-core kernels gives up after a fixed number of polls,
 * raises an abort flag, ORs bit 2 into the status word and returns after
 * freeing its TMEM, so that a wait that can never end leaves the GPU usable.
 * This entry point runs that exit on purpose: one small CTA holds TMEM, waits
 * on an mbarrier nothing arrives on (the MMA thread's spin and the other warps'
 * sleeping wait) with `limit` polls (1 .. 2^24), gives up, ORs 2 into *status
 * (device int32) and adds 1 to *gave_up (device int32) per giving-up warp, 3 in
 * all.  It issues no copy and no MMA, so nothing is in flight when it exits.
 * Enqueued on `stream`; MSA_ERR_INVALID_ARG for null or misaligned pointers or
 * a limit out of range. */
msa_status_t msa_selftest_wait_timeout(uint32_t limit, int32_t* status, int32_t* gave_up,
                                       void* stream);

/* The CUDA error behind the last MSA_ERR_CUDA returned to the calling thread:
 * its cudaError_t value in *code_opt (if not NULL; 0 = none yet) and its
 * description (static storage). */
const char* msa_last_cuda_error(int32_t* code_opt);

/* Human-readable name of a status code (static storage). */
const char* msa_status_string(msa_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
