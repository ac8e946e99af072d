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
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in), so every call looks the address up with
// cudaGetSymbolAddress, with the caller's device current.  The lookup is a
// host-side query, not stream work; the first call on a device also loads the
// library's device code there, so make that first call before any stream
// capture.  Looking the address up on every call (rather than once) keeps it
// right after the device's primary context has been reset and recreated.
//
// Every call clears the part of the array it needs, except the sticky device
// status word, with cudaMemsetAsync on the caller's stream, and then runs the
// ordinary greedy verify on it.  Status bits raised on the device (a timed-out
// wait, an invalid draft token) accumulate until
// spec_verify_greedy_noalloc_read_device_status reads and clears them.  All
// calls share the one array, so two calls whose kernels may overlap on the
// GPU (different streams without ordering between them) race and give wrong
// results: order them on one stream.
#include <cstddef>

#include "spec_verify.h"
#include "sv_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(2) << 20;  // 2 MiB
static_assert(kStaticScratchBytes == SV_NOALLOC_SCRATCH_BYTES,
              "header and library disagree on the scratch size");

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// The control block at the start of every workspace: the sticky status word
// sits between the words that must start each call at zero.
constexpr size_t kFlagsOffset = offsetof(sv::Ctrl, flags);
static_assert(kFlagsOffset + sizeof(unsigned int) <= sizeof(sv::Ctrl), "status word in Ctrl");

// Device address of g_scratch on the current device.
int scratch_address(unsigned char** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SV_ERR_CUDA;
  *out = static_cast<unsigned char*>(p);
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
  unsigned char* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != SV_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kFlagsOffset, st) != cudaSuccess ||
      cudaMemsetAsync(ws + kFlagsOffset + sizeof(unsigned int), 0,
                      need - kFlagsOffset - sizeof(unsigned int), st) != cudaSuccess)
    return SV_ERR_CUDA;
  return spec_verify_greedy(target_logits, t_dtype, t_stride_b, t_stride_pos, draft_tokens, B, k,
                            V, accepted_len, out_tokens, ws, need, stream);
}

extern "C" int spec_verify_greedy_noalloc_read_device_status(uint32_t* flags_host, int clear,
                                                             void* stream) {
  if (!flags_host) return SV_ERR_INVALID_ARG;
  unsigned char* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != SV_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws + kFlagsOffset, sizeof v, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SV_ERR_CUDA;
  *flags_host = v;
  if (clear && cudaMemsetAsync(ws + kFlagsOffset, 0, sizeof v, st) != cudaSuccess)
    return SV_ERR_CUDA;
  return SV_OK;
}
