// noalloc.cu -- pararnn_adjoint_noalloc: the adjoint without a caller-supplied
// workspace.
//
// Some callers cannot hand the library a scratch buffer: they do not own the
// device memory (a framework's caching allocator or a serving process with a
// fixed memory budget owns all of it), or they run on a path where calling
// cudaMalloc -- with its latency and implicit synchronisation -- is not
// acceptable.  For them this entry point runs the same adjoint kernels with
// their scratch in a fixed array compiled into the library, so the call
// allocates nothing.
//
// The array lives in device memory of every GPU that loads the library and
// stays there until the process exits.  It is shared by all calls on that
// device and keeps what the last call left in it.  Nothing a call leaves
// behind can mislead the next one: the look-back adjoint clears its flags on
// the stream at the start of every call, and the whole-sequence adjoint keeps
// its partial sums after the 256-byte header, which it does not touch.  The
// first call on a device also clears the whole array, on the caller's stream
// ahead of that call's kernels.  Calls that overlap on the GPU (different
// streams, or different host threads, without ordering) race on the array and
// must not be made.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = PARARNN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Device-side scratch.  In host code `g_scratch` only names the symbol; its
// device address comes from cudaGetSymbolAddress on the device in question.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Once per device, with that device current: look up the array's address and
// clear it on `stream` (ordered before the kernels the caller enqueues next on
// that stream).  Returns null on failure.
void* scratch_for_current_device(cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    if (cudaMemsetAsync(p, 0, kScratchBytes, stream) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_ptr[dev] = p;
  }
  return g_ptr[dev];
}

}  // namespace

extern "C" int pararnn_adjoint_noalloc(int cell, const void* u, int u_dtype, const float* a,
                                       const float* bias, const float* c0, const float* h0,
                                       const float* c, const float* h, const float* dLdh,
                                       float* du, float* da, float* dbias, float* dc0,
                                       float* dh0, int B, int T, int D, int* status,
                                       pararnn_stream_t stream) {
  // an invalid cell or size (no workspace size) and sizes beyond the built-in
  // scratch are refused before anything else runs
  const size_t need = pararnn_workspace_size(cell, B, T, D, 0, 1);
  if (need == 0) return PARARNN_ERR_INVALID_ARG;
  if (need > kScratchBytes) return PARARNN_ERR_WORKSPACE_TOO_SMALL;
  void* ws = scratch_for_current_device((cudaStream_t)stream);
  if (ws == nullptr) return PARARNN_ERR_CUDA;
  return pararnn_adjoint(cell, u, u_dtype, a, bias, c0, h0, c, h, dLdh, du, da, dbias, dc0, dh0,
                         B, T, D, status, ws, kScratchBytes, stream);
}
