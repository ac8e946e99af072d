// sv_noalloc.cu -- greedy verify for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) on the path
// that runs verify: an allocator hook or memory pool owns every byte of the
// device, the call sits in a real-time loop where an allocation may block or
// fail, or the code must run on a stream whose allocations are forbidden.
// They also cannot keep a workspace of their own.  This entry point gives
// them greedy verify with no allocation at all: its workspace is a fixed,
// file-scope device array that the library carries in its image, so every
// GPU that loads the library holds kStaticScratchBytes of it until the
// process exits.
//
// The first call on each device looks up that array's device address
// (cudaGetSymbolAddress, with the device current) and keeps it; make that
// first call before any stream capture.  Every call clears the part of the
// array it needs (cudaMemsetAsync on the caller's stream) and then runs the
// ordinary greedy verify on it.  All calls share the one array, so two calls
// whose kernels may overlap on the GPU (different streams without ordering
// between them) race and give wrong results: order them on one stream.
#include <mutex>

#include "spec_verify.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(2) << 20;  // 2 MiB
static_assert(kStaticScratchBytes == SV_NOALLOC_SCRATCH_BYTES,
              "header and library disagree on the scratch size");

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_lock;
void* g_scratch_ptr[64] = {};

// Device address of g_scratch on the current device, looked up once.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SV_ERR_CUDA;
  std::lock_guard<std::mutex> guard(g_lock);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SV_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SV_OK;
}

}  // namespace

extern "C" int spec_verify_greedy_noalloc(const void* target_logits, int t_dtype,
                                          int64_t t_stride_b, int64_t t_stride_pos,
                                          const int32_t* draft_tokens, int B, int k, int V,
                                          int32_t* accepted_len, int32_t* out_tokens,
                                          void* stream) {
  const size_t need = spec_verify_workspace_size(B, 1, k, V);
  if (need == 0) return SV_ERR_INVALID_ARG;  // B, k or V outside the limits
  if (need > kStaticScratchBytes) return SV_ERR_WORKSPACE;
  if (B == 0) return SV_OK;
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != SV_OK) return rc;
  if (cudaMemsetAsync(ws, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SV_ERR_CUDA;
  return spec_verify_greedy(target_logits, t_dtype, t_stride_b, t_stride_pos, draft_tokens, B, k,
                            V, accepted_len, out_tokens, ws, need, stream);
}
