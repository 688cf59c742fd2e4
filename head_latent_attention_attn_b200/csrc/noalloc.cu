// noalloc.cu - mla_decode_attn_noalloc: the decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they decode: code running
// inside a memory pool or allocator hook that must not re-enter the allocator, runtimes
// that hand out a fixed memory budget up front, or embedders that forbid device
// allocation after start-up. mla_decode_attn needs a caller-provided workspace for the
// partial results of sequences that are split across CTAs; this entry point instead uses
// a fixed scratch array that lives in the library's own device memory for as long as the
// library is loaded (every GPU that loads the library holds it until process exit).
//
// The array is a file-scope __device__ variable. Host code cannot use its name as a
// device address: on first use on each device the address is looked up with
// cudaGetSymbolAddress (with that device current) and then passed to the kernels.
#include <mutex>

#include "host_common.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = MLA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
mla_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Move the error bits the decode left in the scratch's error word into the caller's word
// and clear the scratch word, so every call starts from a clean word.
__global__ void fold_error_word(int32_t* scratch_word, int32_t* caller_word) {
  const int32_t v = *scratch_word;
  if (v != 0) {
    atomicOr(caller_word, v);
    *scratch_word = 0;
  }
}

}  // namespace

extern "C" size_t mla_decode_workspace_size(const mla_dims*, int32_t, int32_t, int32_t, int32_t);
extern "C" mla_status mla_decode_attn(const mla_dims*, const void*, const void*, int64_t,
                                      const int32_t*, int32_t, const int32_t*, int32_t, int32_t,
                                      int32_t, int32_t, int32_t, void*, size_t, void*, float*,
                                      void*);

// The decode of mla_decode_attn with its workspace carved out of the fixed scratch array.
// The automatic plan is used: it has at most one work range per SM, and no explicit split
// count gives fewer ranges once there are more (sequence, row block) units than SMs, so a
// problem whose automatic plan does not fit is rejected with MLA_ERR_WORKSPACE before
// anything is launched.
extern "C" mla_status mla_decode_attn_noalloc(const mla_dims* dims, const void* q_ext,
                                              const void* cache, int64_t num_pages,
                                              const int32_t* block_table,
                                              int32_t max_pages_per_seq,
                                              const int32_t* seq_lens, int32_t batch,
                                              int32_t q_len, int32_t max_seq_len, int32_t causal,
                                              int32_t* dev_error, void* o_latent, float* lse,
                                              void* stream) {
  if (dev_error == nullptr) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_decode_workspace_size(dims, batch, q_len, max_seq_len, 0);
  if (need == 0 || batch == 0) {
    // invalid or unsupported problem, or nothing to do: report what mla_decode_attn's
    // validation reports (it returns before looking at the workspace and launches nothing)
    return mla_decode_attn(dims, q_ext, cache, num_pages, block_table, max_pages_per_seq,
                           seq_lens, batch, q_len, max_seq_len, causal, 0, nullptr, 0, o_latent,
                           lse, stream);
  }
  if (need > kScratchBytes) return MLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  mla_status st = scratch_address(&scratch);
  if (st != MLA_OK) return st;
  // The scratch is used exactly like a workspace: its first int32 is the decode's error
  // word, the rest is fully rewritten by every call.
  unsigned char* ws = static_cast<unsigned char*>(scratch);
  st = mla_decode_attn(dims, q_ext, cache, num_pages, block_table, max_pages_per_seq, seq_lens,
                       batch, q_len, max_seq_len, causal, 0, ws, round256(need), o_latent, lse,
                       stream);
  if (st != MLA_OK && st != MLA_ERR_CUDA) return st;   // rejected before any launch
  // After any launch (even one followed by a failed launch) move the bits the decode left in
  // the scratch's error word into the caller's word and clear it, so no call inherits them.
  fold_error_word<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<int32_t*>(ws),
                                                                  dev_error);
  const cudaError_t le = cudaGetLastError();
  if (st != MLA_OK) return st;
  return le == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
