// C ABI of libmsa: argument checks, workspace layout and the launch sequence.
// Declarations and the contract of every entry point are in include/msa.h.
#include <math.h>
#include <string.h>

#include "../../include/msa.h"
#include "internal.h"

using msa::Problem;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_divides_128(int g) { return g >= 1 && g <= 128 && (128 % g) == 0; }

// Shape checks shared by every entry point.
msa_status_t resolve(const msa_problem_t* p, Problem* P) {
  if (!p) return MSA_ERR_INVALID_ARG;
  if (p->index_dtype != 0 && !((p->index_dtype == MSA_FP8_E4M3 || p->index_dtype == MSA_NVFP4) &&
                                p->dtype == MSA_BF16))
    return MSA_ERR_INVALID_ARG;
  if (p->index_dtype == MSA_NVFP4 && (!p->q_idx_scale || !p->k_idx_scale))
    return MSA_ERR_INVALID_ARG;
  if (p->qk_dtype != 0 && !(p->qk_dtype == MSA_FP8_E4M3 && p->dtype == MSA_BF16))
    return MSA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->q_len < 0 || p->kv_len < 1 || p->q_pos0 < 0) return MSA_ERR_INVALID_ARG;
  if (p->q_pos0 + p->q_len > p->kv_len) return MSA_ERR_INVALID_ARG;
  if (p->num_kv_heads < 1 || p->num_q_heads < 1 || p->num_q_heads % p->num_kv_heads != 0)
    return MSA_ERR_INVALID_ARG;
  if (p->block_size < 1 || p->top_k < 1 || p->head_dim < 1 || p->index_dim < 1)
    return MSA_ERR_INVALID_ARG;
  if (p->dtype != MSA_BF16 && p->dtype != MSA_F32) return MSA_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.0f) || isinf(p->softmax_scale)) return MSA_ERR_INVALID_ARG;
  const int G = p->num_q_heads / p->num_kv_heads;
  // 128-token blocks on every kernel; 64 and 32 on the CUDA-core kernels (the
  // tensor-core kernels tile one 128-key block per MMA and say so)
  if (p->block_size != 128 && p->block_size != 64 && p->block_size != 32)
    return MSA_ERR_UNSUPPORTED;
  if (p->top_k > 32) return MSA_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (p->index_dim != 32 && p->index_dim != 64 && p->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (!pow2_divides_128(G)) return MSA_ERR_UNSUPPORTED;
  const long long T = (long long)p->batch * p->q_len;
  if (T * 32 >= (1LL << 31)) return MSA_ERR_UNSUPPORTED;                      // entry packing
  if ((long long)p->num_kv_heads * T * p->top_k >= (1LL << 31)) return MSA_ERR_UNSUPPORTED;
  if ((long long)p->batch * p->kv_len >= (1LL << 31)) return MSA_ERR_UNSUPPORTED;
  P->B = p->batch;
  P->Sq = p->q_len;
  P->Skv = p->kv_len;
  P->Hq = p->num_q_heads;
  P->Hkv = p->num_kv_heads;
  P->D = p->head_dim;
  P->DI = p->index_dim;
  P->Bk = p->block_size;
  P->K = p->top_k;
  P->G = G;
  P->T = int(T);
  P->nblk = (p->kv_len + p->block_size - 1) / p->block_size;
  P->nqc = (p->q_len + msa::kQueryChunk - 1) / msa::kQueryChunk;
  if (P->nqc < 1) P->nqc = 1;
  P->qpt = 128 / G;
  P->q_pos0 = p->q_pos0;
  P->scale = p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / sqrtf((float)p->head_dim);
  P->f32 = p->dtype == MSA_F32;
  P->idx8 = p->index_dtype == MSA_FP8_E4M3;
  P->idx4 = p->index_dtype == MSA_NVFP4;
  P->qsc = P->idx4 ? p->q_idx_scale : nullptr;
  P->ksc = P->idx4 ? p->k_idx_scale : nullptr;
  P->qk8 = p->qk_dtype == MSA_FP8_E4M3;
  if (p->num_pages < 0 || (p->num_pages > 0 && !p->block_table)) return MSA_ERR_INVALID_ARG;
  if (p->num_pages > 0 && p->block_size != 128) return MSA_ERR_UNSUPPORTED;  // page = block
  P->table = p->num_pages > 0 ? p->block_table : nullptr;
  P->pages = p->num_pages;
  P->kv_rows = P->table ? (long long)P->pages * P->Bk : (long long)P->B * P->Skv;
  if (P->kv_rows >= (1LL << 31)) return MSA_ERR_UNSUPPORTED;
  P->nlists = (long long)P->B * P->Hkv * P->nqc * P->nblk;
  if (P->nlists + 1 >= (1LL << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// Workspace layout (each region 256-byte aligned, in this order).
struct Layout {
  size_t status, bmax, q2k, counts, cursor, list_off, tile_off, entries, pos, tiles, seg_sums,
      part_o, part_lse, kl_rows, kl_ds, idx_q, idx_k, total;
};

// NVFP4 index tensors that the key-streaming kernel does not take are decoded
// to bf16 in the workspace first; the index branch then runs on this problem.
bool nvfp4_decoded(const Problem& P) { return P.idx4 && !msa::nvfp4_keys_supported(P); }

Problem index_problem(const Problem& P) {
  Problem Q = P;
  if (nvfp4_decoded(P)) {
    Q.idx4 = false;
    Q.qsc = Q.ksc = nullptr;
  }
  return Q;
}

Layout layout(const Problem& P, int op) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align_up(bytes); return o; };
  const size_t T = size_t(P.T);
  const size_t esz = P.f32 ? 4 : 2;
  L.status = take(sizeof(int32_t));
  const bool sel = op == MSA_OP_SELECT || op == MSA_OP_FORWARD;
  const bool att = op == MSA_OP_ATTEND || op == MSA_OP_FORWARD;
  const bool kl = op == MSA_OP_INDEX_KL;
  const Problem PI = index_problem(P);
  // the index branch's scratch: partial selection lists when the selection is
  // fused into the index kernel, else the block maxima
  L.bmax = sel ? take(msa::index_select_fused_supported(PI)
                          ? msa::index_select_cand_bytes(PI)
                          : size_t(P.Hkv) * T * P.nblk * sizeof(float))
               : 0;
  if (sel && nvfp4_decoded(P)) {  // bf16 copies of q_idx and k_idx
    L.idx_q = take(T * P.Hkv * P.DI * 2);
    L.idx_k = take(size_t(P.kv_rows) * P.DI * 2);
  }
  L.q2k = op == MSA_OP_FORWARD ? take(size_t(P.Hkv) * T * P.K * sizeof(int32_t)) : 0;
  if (att || kl) {
    L.counts = take(size_t(P.nlists) * 4);
    L.cursor = take(size_t(P.nlists) * 4);
    L.list_off = take(size_t(P.nlists + 1) * 4);
    L.tile_off = take(size_t(P.nlists + 1) * 4);
    L.entries = take(size_t(P.Hkv) * T * P.K * 4);
    L.pos = take(size_t(P.Hkv) * T * P.K * 4);
    L.seg_sums = take(size_t((P.nlists + 2047) / 2048) * 8);
  }
  if (kl) {
    L.kl_rows = take(size_t(P.Hkv) * T * sizeof(float));
    L.kl_ds = take(size_t(P.Hkv) * T * P.K * P.Bk * sizeof(float));
  }
  if (att) {
    L.tiles = take(size_t(msa::max_tiles(P)) * sizeof(msa::TileRec));
    // one partial state per (entry, head of the group): Hkv*T*K*G = T*Hq*K rows
    L.part_o = take(T * P.Hq * P.K * size_t(P.D) * esz);
    L.part_lse = take(T * P.Hq * P.K * sizeof(float));
  }
  L.total = off;
  return L;
}

// The CUDA error behind the last MSA_ERR_CUDA of this thread (msa_last_cuda_error).
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

msa_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MSA_OK;
  g_last_cuda_error = e;
  return MSA_ERR_CUDA;
}

// Optional stage events (msa_set_stage_events).  Every entry point restarts
// the numbering (stage_begin) so that each call records its own stages.
cudaEvent_t const* g_events = nullptr;
int g_nevents = 0;
int g_next = 0;

void stage_begin() { g_next = 0; }

void stage_mark(cudaStream_t s) {
  if (g_events && g_next < g_nevents) cudaEventRecord(g_events[g_next++], s);
}

template <typename P_>
P_* at(void* ws, size_t off) { return reinterpret_cast<P_*>(static_cast<char*>(ws) + off); }

msa_status_t check_ws(const Problem& P, int op, const void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MSA_ERR_INVALID_ARG;
  if (ws_bytes < layout(P, op).total) return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

msa::Lists lists_of(void* ws, const Layout& L) {
  return msa::Lists{at<int32_t>(ws, L.counts), at<int32_t>(ws, L.cursor),
                    at<int32_t>(ws, L.list_off), at<int32_t>(ws, L.tile_off),
                    at<int32_t>(ws, L.entries), at<int32_t>(ws, L.pos),
                    at<int32_t>(ws, L.tiles), at<int32_t>(ws, L.seg_sums)};
}

// run_select's top-k also writes the block -> query lists (lists != nullptr):
// msa_forward on one query row per sequence whose rows all keep top_k blocks.
msa_status_t run_select(const Problem& P0, const void* q_idx, const void* k_idx, int32_t* q2k,
                        float* bscores, void* ws, cudaStream_t s,
                        const msa::Lists* lists = nullptr) {
  const Layout L = layout(P0, MSA_OP_SELECT);
  float* bmax = bscores ? bscores : at<float>(ws, L.bmax);
  cudaError_t e = msa::launch_check_table(P0, at<int32_t>(ws, L.status), s);
  // NVFP4 codes: the key-streaming kernel reads them as they are; otherwise
  // they are decoded (exactly) to bf16 and the bf16 kernels run on the copies
  if (e == cudaSuccess && nvfp4_decoded(P0)) {
    e = msa::launch_dequant_nvfp4(q_idx, P0.qsc, at<void>(ws, L.idx_q),
                                  (long long)P0.T * P0.Hkv, P0.DI, s);
    if (e == cudaSuccess)
      e = msa::launch_dequant_nvfp4(k_idx, P0.ksc, at<void>(ws, L.idx_k), P0.kv_rows, P0.DI, s);
    q_idx = at<void>(ws, L.idx_q);
    k_idx = at<void>(ws, L.idx_k);
  }
  const Problem P = index_problem(P0);
  if (!bscores && msa::index_select_fused_supported(P)) {
    // selection streamed inside the index kernel, then a merge of the partial lists
    if (e == cudaSuccess) {
      e = msa::launch_index_select(P, q_idx, k_idx, at<void>(ws, L.bmax),
                                   at<int32_t>(ws, L.status), s);
      stage_mark(s);
    }
    if (e == cudaSuccess) {
      e = msa::launch_select_merge(P, at<void>(ws, L.bmax), q2k, s);
      stage_mark(s);
    }
    return cuda_status(e);
  }
  if (bscores && e == cudaSuccess)
    e = msa::launch_fill(bscores, size_t(P.Hkv) * P.T * P.nblk, -INFINITY, s);
  if (e == cudaSuccess) {
    int32_t* status = at<int32_t>(ws, L.status);
    e = P.idx4                           ? msa::launch_index_nvfp4_keys(P, q_idx, k_idx, bmax, s)
        : msa::index_tc_supported(P)     ? msa::launch_index_tc(P, q_idx, k_idx, bmax, status, s)
        : msa::index_decode_supported(P) ? msa::launch_index_decode(P, q_idx, k_idx, bmax, status, s)
                                         : msa::launch_index_simt(P, q_idx, k_idx, bmax, s);
    stage_mark(s);
  }
  if (e == cudaSuccess) {
    e = lists ? msa::launch_topk_lists(P, bmax, q2k, *lists, s) : msa::launch_topk(P, bmax, q2k, s);
    stage_mark(s);
  }
  return cuda_status(e);
}

// lists_ready: the top-k kernel of the same call has written the lists already.
msa_status_t run_attend(const Problem& P, const void* q, const void* k, const void* v,
                        const int32_t* q2k, void* out, float* lse, void* ws, const Layout& L,
                        cudaStream_t s, bool lists_ready = false) {
  const msa::Lists lists = lists_of(ws, L);
  msa::Partials part{at<void>(ws, L.part_o), at<float>(ws, L.part_lse)};
  const bool tc = msa::attn_tc_supported(P);
  cudaError_t e = msa::launch_check_table(P, at<int32_t>(ws, L.status), s);
  if (e != cudaSuccess || lists_ready) {
  } else if (msa::lists_direct(P)) {
    e = msa::launch_lists_direct(P, q2k, lists, at<int32_t>(ws, L.status), s);
  } else {
    e = msa::launch_invert(P, q2k, lists, at<int32_t>(ws, L.status), s);
    if (e == cudaSuccess && tc) e = msa::launch_tile_records(P, lists, s);
  }
  stage_mark(s);
  if (e == cudaSuccess) {
    e = tc ? msa::launch_attn_tc(P, q, k, v, lists, part, at<int32_t>(ws, L.status), s)
            : msa::launch_attn_simt(P, q, k, v, lists, part, s);
    stage_mark(s);
  }
  if (e == cudaSuccess) {
    e = msa::launch_combine(P, lists.pos, part, out, lse, at<int32_t>(ws, L.status), s);
    stage_mark(s);
  }
  return cuda_status(e);
}

// Index branch, selection and main branch of one resolved problem whose
// workspace is checked and whose status word is already cleared; q2k is the
// caller's buffer or, when NULL, the workspace's own.
msa_status_t forward_one(const Problem& P, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, void* out, float* lse,
                         int32_t* q2k_opt, void* ws, cudaStream_t s) {
  const Layout L = layout(P, MSA_OP_FORWARD);
  int32_t* q2k = q2k_opt ? q2k_opt : at<int32_t>(ws, L.q2k);
  // the select stage only needs the status word and bmax, which sit at the same
  // offsets in the forward layout
  const bool topk_lists =
      msa::topk_writes_lists(P) && !msa::index_select_fused_supported(index_problem(P));
  const msa::Lists lists = lists_of(ws, L);
  msa_status_t st = run_select(P, q_idx, k_idx, q2k, nullptr, ws, s, topk_lists ? &lists : nullptr);
  if (st != MSA_OK) return st;
  return run_attend(P, q, k, v, q2k, out, lse, ws, L, s, topk_lists);
}

// A packed variable-length batch as runs of consecutive sequences with the
// same (query rows, keys): each run is one fixed-length batched problem, since
// equal-length sequences packed back to back are exactly the [batch, len, ...]
// layout.  Sequences without query rows are left out (they end a run).
struct Run {
  int b0, nseq, nq, nk;
};

constexpr int kMaxVarlenSeqs = 1 << 20;

msa_status_t varlen_runs(const msa_problem_t* p, const int32_t* cu_q, const int32_t* cu_k,
                         Run* runs, int* nruns, long long* total_q) {
  if (!p || !cu_q || !cu_k || p->batch < 1 || p->batch > kMaxVarlenSeqs)
    return MSA_ERR_INVALID_ARG;
  if (p->num_pages != 0) return MSA_ERR_UNSUPPORTED;
  if (cu_q[0] != 0 || cu_k[0] != 0) return MSA_ERR_INVALID_ARG;
  int n = 0;
  for (int b = 0; b < p->batch; ++b) {
    const long long nq = (long long)cu_q[b + 1] - cu_q[b];
    const long long nk = (long long)cu_k[b + 1] - cu_k[b];
    if (nq < 0 || nk < 0 || nq > nk) return MSA_ERR_INVALID_ARG;
    if (nq == 0) continue;
    if (n > 0 && runs[n - 1].b0 + runs[n - 1].nseq == b && runs[n - 1].nq == nq &&
        runs[n - 1].nk == nk) {
      ++runs[n - 1].nseq;
    } else {
      runs[n++] = Run{b, 1, int(nq), int(nk)};
    }
  }
  *nruns = n;
  *total_q = cu_q[p->batch];
  return MSA_OK;
}

// The fixed-length problem of one run.
msa_problem_t run_problem(const msa_problem_t* p, const Run& r) {
  msa_problem_t q = *p;
  q.batch = r.nseq;
  q.q_len = r.nq;
  q.kv_len = r.nk;
  q.q_pos0 = r.nk - r.nq;  // a sequence's query rows are its last tokens
  return q;
}

// Runs of a packed batch, resolved; the run list lives on the heap (one entry
// per sequence at most).
struct VarlenPlan {
  Run* runs = nullptr;
  int n = 0;
  long long total_q = 0;
  size_t ws = 0;  // workspace of the largest run (runs reuse it one after another)
  ~VarlenPlan() { delete[] runs; }
};

msa_status_t plan_varlen(const msa_problem_t* p, const int32_t* cu_q, const int32_t* cu_k,
                         VarlenPlan* plan) {
  if (!p || p->batch < 1 || p->batch > kMaxVarlenSeqs) return MSA_ERR_INVALID_ARG;
  plan->runs = new Run[p->batch];
  msa_status_t st = varlen_runs(p, cu_q, cu_k, plan->runs, &plan->n, &plan->total_q);
  if (st != MSA_OK) return st;
  plan->ws = align_up(sizeof(int32_t));
  for (int i = 0; i < plan->n; ++i) {
    const msa_problem_t rp = run_problem(p, plan->runs[i]);
    Problem P;
    if ((st = resolve(&rp, &P)) != MSA_OK) return st;
    const size_t w = layout(P, MSA_OP_FORWARD).total;
    if (w > plan->ws) plan->ws = w;
  }
  return MSA_OK;
}

}  // namespace

namespace msa {
msa_status_t resolve_problem(const msa_problem_t* p, Problem* P) { return resolve(p, P); }
msa_status_t status_of(cudaError_t e) { return cuda_status(e); }
}  // namespace msa

extern "C" {

size_t msa_workspace_size(const msa_problem_t* p, int32_t op) {
  Problem P;
  if (resolve(p, &P) != MSA_OK || op < MSA_OP_SELECT || op > MSA_OP_INDEX_KL) return 0;
  return layout(P, op).total;
}

msa_status_t msa_select(const msa_problem_t* p, const void* q_idx, const void* k_idx,
                        int32_t* q2k, float* block_scores_opt, void* ws, size_t ws_bytes,
                        void* stream) {
  Problem P;
  msa_status_t st = resolve(p, &P);
  if (st != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;  // nothing to do; empty tensors may carry null pointers
  if (!q_idx || !k_idx || !q2k) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q2k) ||
      (block_scores_opt && !aligned16(block_scores_opt)))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(P, MSA_OP_SELECT, ws, ws_bytes)) != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;
  if (msa_status_t cst = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), (cudaStream_t)stream)))
    return cst;
  stage_begin();
  return run_select(P, q_idx, k_idx, q2k, block_scores_opt, ws, (cudaStream_t)stream);
}

msa_status_t msa_attend(const msa_problem_t* p, const void* q, const void* k, const void* v,
                        const int32_t* q2k, void* out, float* lse_opt, void* ws,
                        size_t ws_bytes, void* stream) {
  Problem P;
  msa_status_t st = resolve(p, &P);
  if (st != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;  // nothing to do; empty tensors may carry null pointers
  if (!q || !k || !v || !q2k || !out) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q2k) || !aligned16(out) ||
      (lse_opt && !aligned16(lse_opt)))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(P, MSA_OP_ATTEND, ws, ws_bytes)) != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;
  if (msa_status_t cst = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), (cudaStream_t)stream)))
    return cst;
  stage_begin();
  return run_attend(P, q, k, v, q2k, out, lse_opt, ws, layout(P, MSA_OP_ATTEND),
                    (cudaStream_t)stream);
}

msa_status_t msa_forward(const msa_problem_t* p, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, void* out, float* lse_opt,
                         int32_t* q2k_opt, void* ws, size_t ws_bytes, void* stream) {
  Problem P;
  msa_status_t st = resolve(p, &P);
  if (st != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;  // nothing to do; empty tensors may carry null pointers
  if (!q || !k || !v || !q_idx || !k_idx || !out) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) ||
      !aligned16(k_idx) || !aligned16(out) || (lse_opt && !aligned16(lse_opt)) ||
      (q2k_opt && !aligned16(q2k_opt)))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(P, MSA_OP_FORWARD, ws, ws_bytes)) != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (msa_status_t cst = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), s))) return cst;
  stage_begin();
  return forward_one(P, q, k, v, q_idx, k_idx, out, lse_opt, q2k_opt, ws, s);
}

size_t msa_varlen_workspace_size(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                 const int32_t* cu_seqlens_k) {
  VarlenPlan plan;
  if (plan_varlen(p, cu_seqlens_q, cu_seqlens_k, &plan) != MSA_OK) return 0;
  return plan.ws;
}

int32_t msa_varlen_launch_count(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k) {
  VarlenPlan plan;
  if (plan_varlen(p, cu_seqlens_q, cu_seqlens_k, &plan) != MSA_OK) return 0;
  int32_t n = 0;
  for (int i = 0; i < plan.n; ++i) {
    const msa_problem_t rp = run_problem(p, plan.runs[i]);
    n += msa_launch_count(&rp, MSA_OP_FORWARD);
  }
  return n;  // the q2k copies (q2k_opt) are memory copies, not kernel launches
}

msa_status_t msa_forward_varlen(const msa_problem_t* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, const void* q, const void* k,
                                const void* v, const void* q_idx, const void* k_idx, void* out,
                                float* lse_opt, int32_t* q2k_opt, void* ws, size_t ws_bytes,
                                void* stream) {
  VarlenPlan plan;
  msa_status_t st = plan_varlen(p, cu_seqlens_q, cu_seqlens_k, &plan);
  if (st != MSA_OK) return st;
  if (plan.total_q == 0) return MSA_OK;  // no query row: nothing to do
  if (!q || !k || !v || !q_idx || !k_idx || !out) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) ||
      !aligned16(k_idx) || !aligned16(out) || (lse_opt && !aligned16(lse_opt)) ||
      (q2k_opt && !aligned16(q2k_opt)))
    return MSA_ERR_INVALID_ARG;
  // the runs' log-normalisers start at row offsets of num_q_heads floats
  if (lse_opt && p->num_q_heads % 4 != 0) return MSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MSA_ERR_INVALID_ARG;
  if (ws_bytes < plan.ws) return MSA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  // one status word for the whole call: the runs OR their flags into it
  if (msa_status_t cst = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), s))) return cst;
  stage_begin();
  const size_t esz = p->dtype == MSA_F32 ? 4 : 2;
  const size_t esz_qk = p->qk_dtype == MSA_FP8_E4M3 ? 1 : esz;
  const size_t esz_idx = p->index_dtype == MSA_FP8_E4M3 ? 1 : esz;
  const size_t qrow = size_t(p->num_q_heads) * p->head_dim;   // elements per query row
  const size_t krow = size_t(p->num_kv_heads) * p->head_dim;  // per key row
  for (int i = 0; i < plan.n; ++i) {
    const Run& r = plan.runs[i];
    const msa_problem_t rp = run_problem(p, r);
    Problem P;
    if ((st = resolve(&rp, &P)) != MSA_OK) return st;
    const size_t q0 = size_t(cu_seqlens_q[r.b0]), k0 = size_t(cu_seqlens_k[r.b0]);
    const char* qb = static_cast<const char*>(q) + q0 * qrow * esz_qk;
    const char* kb = static_cast<const char*>(k) + k0 * krow * esz_qk;
    const char* vb = static_cast<const char*>(v) + k0 * krow * esz;
    const char* qib = static_cast<const char*>(q_idx) + q0 * p->num_kv_heads * p->index_dim * esz_idx;
    const char* kib = static_cast<const char*>(k_idx) + k0 * p->index_dim * esz_idx;
    char* ob = static_cast<char*>(out) + q0 * qrow * esz;
    float* lb = lse_opt ? lse_opt + q0 * p->num_q_heads : nullptr;
    if ((st = forward_one(P, qb, kb, vb, qib, kib, ob, lb, nullptr, ws, s)) != MSA_OK) return st;
    if (q2k_opt) {
      // the run's [Hkv, rows, top_k] selection into the packed [Hkv, total_q, top_k]
      const Layout L = layout(P, MSA_OP_FORWARD);
      const size_t w = size_t(P.T) * P.K * sizeof(int32_t);
      if (msa_status_t cst = cuda_status(cudaMemcpy2DAsync(
              q2k_opt + q0 * P.K, size_t(plan.total_q) * P.K * sizeof(int32_t),
              at<int32_t>(ws, L.q2k), w, w, size_t(P.Hkv), cudaMemcpyDeviceToDevice, s)))
        return cst;
    }
  }
  return MSA_OK;
}

msa_status_t msa_index_kl(const msa_problem_t* p, const void* q, const void* k,
                          const void* q_idx, const void* k_idx, const int32_t* q2k,
                          float* loss, float* dq_idx, float* dk_idx, void* ws, size_t ws_bytes,
                          void* stream) {
  Problem P;
  msa_status_t st = resolve(p, &P);
  if (st != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;  // no (row, group) pair: nothing to average
  if (!msa::index_kl_supported(P)) return MSA_ERR_UNSUPPORTED;
  if (!q || !k || !q_idx || !k_idx || !q2k || !loss || !dq_idx || !dk_idx)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_idx) || !aligned16(k_idx) ||
      !aligned16(q2k) || !aligned16(dq_idx) || !aligned16(dk_idx) ||
      (reinterpret_cast<uintptr_t>(loss) & 3u) != 0)
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(P, MSA_OP_INDEX_KL, ws, ws_bytes)) != MSA_OK) return st;
  const Layout L = layout(P, MSA_OP_INDEX_KL);
  cudaStream_t s = (cudaStream_t)stream;
  if (msa_status_t cst = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), s))) return cst;
  msa::Lists lists{at<int32_t>(ws, L.counts), at<int32_t>(ws, L.cursor),
                   at<int32_t>(ws, L.list_off), at<int32_t>(ws, L.tile_off),
                   at<int32_t>(ws, L.entries), at<int32_t>(ws, L.pos), nullptr,
                   at<int32_t>(ws, L.seg_sums)};
  int32_t* status = at<int32_t>(ws, L.status);
  cudaError_t e = msa::launch_check_table(P, status, s);
  if (e == cudaSuccess) e = msa::launch_invert(P, q2k, lists, status, s);
  if (e == cudaSuccess)
    e = msa::launch_index_kl(P, q, k, q_idx, k_idx, q2k, lists, at<float>(ws, L.kl_rows),
                             at<float>(ws, L.kl_ds), loss, dq_idx, dk_idx, status, s);
  return cuda_status(e);
}

msa_status_t msa_device_status(const void* ws, int32_t* code, void* stream) {
  if (!ws || !code) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t h = 0;
  if (msa_status_t cst = cuda_status(cudaMemcpyAsync(&h, ws, sizeof(int32_t),
                                                     cudaMemcpyDeviceToHost, s)))
    return cst;
  if (msa_status_t cst = cuda_status(cudaStreamSynchronize(s))) return cst;
  *code = h;
  return h == 0 ? MSA_OK : MSA_ERR_DEVICE;
}

int32_t msa_set_stage_events(void* const* events, int32_t n) {
  g_events = reinterpret_cast<cudaEvent_t const*>(events);
  g_nevents = events ? n : 0;
  g_next = 0;
  return 5;
}

int32_t msa_launch_count(const msa_problem_t* p, int32_t op) {
  Problem P;
  if (resolve(p, &P) != MSA_OK || P.T == 0) return 0;
  const int chk = P.table ? 1 : 0;                  // block table check (paged)
  const int sel = chk + 2 + (nvfp4_decoded(P) ? 2 : 0);  // (NVFP4 decode x 2) index + top-k
  // lists (+ tile records on the tensor-core path) + attention + combine
  const int att = chk +
                  (msa::lists_direct(P) ? 1
                                        : msa::kLaunchesInvert + (msa::attn_tc_supported(P) ? 1 : 0)) +
                  2;
  switch (op) {
    case MSA_OP_SELECT: return sel;
    case MSA_OP_ATTEND: return att;
    case MSA_OP_FORWARD:
      // the decode top-k writes the lists itself (one launch fewer)
      return sel + att - (msa::topk_writes_lists(P) &&
                          !msa::index_select_fused_supported(index_problem(P)));
    case MSA_OP_INDEX_KL: return chk + msa::kLaunchesInvert + 3;  // lists, rows, dk, sum
  }
  return 0;
}

const char* msa_kernel_path(const msa_problem_t* p, int32_t op) {
  Problem P;
  if (resolve(p, &P) != MSA_OK) return "invalid";
  const bool atc = msa::attn_tc_supported(P);
  const Problem PI = index_problem(P);
  const int ik = PI.idx4 ? 3
                 : msa::index_tc_supported(PI) ? 0 : msa::index_decode_supported(PI) ? 1 : 2;
  static const char* sel[4] = {"index:tc", "index:stream", "index:simt", "index:nvfp4-keys"};
  static const char* fwd[4][2] = {{"index:tc attn:simt", "index:tc attn:tc"},
                                  {"index:stream attn:simt", "index:stream attn:tc"},
                                  {"index:simt attn:simt", "index:simt attn:tc"},
                                  {"index:nvfp4-keys attn:simt", "index:nvfp4-keys attn:tc"}};
  switch (op) {
    case MSA_OP_SELECT: return sel[ik];
    case MSA_OP_ATTEND: return atc ? "attn:tc" : "attn:simt";
    case MSA_OP_FORWARD: return fwd[ik][atc ? 1 : 0];
    case MSA_OP_INDEX_KL: return "kl:simt";
  }
  return "invalid";
}

const char* msa_last_cuda_error(int32_t* code_opt) {
  if (code_opt) *code_opt = int32_t(g_last_cuda_error);
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char* msa_status_string(msa_status_t s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG: null/misaligned pointer or bad shape";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED: shape outside the kernels' coverage";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE: workspace too small";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA: CUDA launch or call failed";
    case MSA_ERR_DEVICE: return "MSA_ERR_DEVICE: invalid q2k entry seen on the device";
    case MSA_ERR_TOO_LARGE:
      return "MSA_ERR_TOO_LARGE: block maxima exceed the 4 MiB static scratch of "
             "msa_select_static";
  }
  return "MSA_ERR_UNKNOWN";
}

}  // extern "C"
