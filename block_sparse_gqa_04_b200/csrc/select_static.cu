// msa_select_static: the index branch (block maxima + top-k selection) with
// its scratch in a fixed device buffer of this library instead of a caller
// workspace, so the call allocates nothing and takes no workspace argument.
//
// It exists for callers that cannot hand the library device memory: a host
// runtime that has reserved all of the device's memory up front (for example
// a decode loop whose KV-cache pool owns the whole device) and has no
// allocator left to lend, or a plain C caller that holds no device allocator.
// The pages describe no such entry point; it runs the same kernels as
// msa_select.
//
// Scratch: one file-scope device array of kScratchBytes, 256-byte aligned:
//   [0, 256)                 status word (int32), cleared by every call
//   [256, 256 + 4 MiB)       block maxima [num_kv_heads, batch*q_len, nblk] fp32
// Only the status word must start at zero (the index kernels OR failure bits
// into it); every block maximum that the top-k kernel reads is written by the
// index kernel of the same call first.
#include <mutex>

#include "../../include/msa.h"
#include "internal.h"

namespace {

constexpr size_t kStatusBytes = 256;
constexpr size_t kMaxBmaxBytes = size_t(4) << 20;
constexpr size_t kScratchBytes = kStatusBytes + kMaxBmaxBytes;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Address of g_scratch on the current device.  Looked up once per device, with
// that device current, on the first call that reaches this point.
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" msa_status_t msa_select_static(const msa_problem_t* p, const void* q_idx,
                                          const void* k_idx, int32_t* q2k,
                                          int32_t* device_status_opt, void* stream) {
  msa::Problem P;
  msa_status_t st = msa::resolve_problem(p, &P);
  if (st != MSA_OK) return st;
  if (P.T == 0) return MSA_OK;  // nothing to do; empty tensors may carry null pointers
  if (!q_idx || !k_idx || !q2k) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q2k) ||
      (device_status_opt && (reinterpret_cast<uintptr_t>(device_status_opt) & 3u) != 0))
    return MSA_ERR_INVALID_ARG;
  const size_t bmax_bytes = size_t(P.Hkv) * size_t(P.T) * size_t(P.nblk) * sizeof(float);
  if (bmax_bytes > kMaxBmaxBytes) return MSA_ERR_TOO_LARGE;
  // NVFP4 only where the key-streaming kernel reads the codes directly (the
  // other index kernels need a bf16 copy, which has no room here)
  if (P.idx4 && !msa::nvfp4_keys_supported(P)) return MSA_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if (msa_status_t cst = msa::status_of(scratch_on_current_device(&scratch))) return cst;
  int32_t* status = static_cast<int32_t*>(scratch);
  float* bmax = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kStatusBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = msa::launch_check_table(P, status, s);
  if (e == cudaSuccess)
    e = P.idx4                           ? msa::launch_index_nvfp4_keys(P, q_idx, k_idx, bmax, s)
        : msa::index_tc_supported(P)     ? msa::launch_index_tc(P, q_idx, k_idx, bmax, status, s)
        : msa::index_decode_supported(P) ? msa::launch_index_decode(P, q_idx, k_idx, bmax, status, s)
                                         : msa::launch_index_simt(P, q_idx, k_idx, bmax, s);
  if (e == cudaSuccess) e = msa::launch_topk(P, bmax, q2k, s);
  if (e == cudaSuccess && device_status_opt)
    e = cudaMemcpyAsync(device_status_opt, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
  return msa::status_of(e);
}
