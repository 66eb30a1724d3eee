// af_noalloc.cu -- af_forward_noalloc: the forward pass of one AF block for
// callers that must not allocate device memory.
//
// Some hosts of this library own all device memory themselves and forbid any
// allocation by the code they call: an application that reserved the GPU's
// memory up front with its own allocator, a plugin inside an inference server
// that only hands its plugins input and output buffers, or a certified
// real-time program that allows no allocation after start-up.  Such a caller
// cannot provide af_forward's workspace.  This entry point takes only the
// inputs and outputs and runs in a scratch array that lives in the library
// itself: a file-scope device array of kScratchBytes (32 MiB), which every GPU
// that loads libaf.so holds until the process exits.
//
// On its first call on a device the entry point looks up the array's device
// address (cudaGetSymbolAddress, with that device current); make that first
// call before any stream capture.  All calls share the one array and the
// array keeps the previous call's contents, so two calls whose work overlaps
// on the GPU (different streams, or different host threads) race and corrupt
// each other's results: serialise them.  Nothing here calls cudaMalloc,
// cudaFree or any allocating routine; the kernels are launched directly on the
// caller's stream.
#include <cuda_runtime.h>
#include <stdio.h>

#include "../../include/af.h"
#include "af_kernels.h"

namespace af {
af_status forward_direct(const af_model* m, const float* x, int batch, int L, af_dir dir, float* z,
                         float* logdet, void* ws, size_t ws_bytes, cudaStream_t st);
af_status check_call_device(const af_model* m, cudaStream_t st);
void set_error_text(const char* msg);
}  // namespace af

namespace {

constexpr size_t kScratchBytes = (size_t)32 << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

void* g_scratch_addr[kMaxDevices];   // the array's device address, per device

}  // namespace

extern "C" af_status af_forward_noalloc(const af_model* m, const float* x, int batch, int L, af_dir dir, float* z,
                                        float* logdet, void* stream) {
  if (!m || !x || !z || !logdet || x == z) {
    af::set_error_text("af_forward_noalloc: null model/x/z/logdet, or x aliases z");
    return AF_ERR_ARG;
  }
  const size_t need = af_workspace_bytes(m, batch, L, L);
  if (!need) {
    af::set_error_text("af_forward_noalloc: bad batch or L for this model");
    return AF_ERR_ARG;
  }
  if (need > kScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof msg,
             "af_forward_noalloc: this call needs %zu bytes of scratch, more than the library's fixed %zu; "
             "use af_forward with a workspace",
             need, kScratchBytes);
    af::set_error_text(msg);
    return AF_ERR_WORKSPACE;
  }
  // the scratch used is the current device's: the model's weights and the
  // stream must be on that device too
  if (af_status s = af::check_call_device(m, (cudaStream_t)stream)) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    af::set_error_text("af_forward_noalloc: no usable current CUDA device");
    return AF_ERR_CUDA;
  }
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      char msg[200];
      snprintf(msg, sizeof msg, "af_forward_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      af::set_error_text(msg);
      return AF_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  // the control block at the head of the scratch starts from zero on every call
  if (cudaMemsetAsync(g_scratch_addr[dev], 0, 256, (cudaStream_t)stream) != cudaSuccess) {
    af::set_error_text("af_forward_noalloc: clearing the control block failed");
    return AF_ERR_CUDA;
  }
  return af::forward_direct(m, x, batch, L, dir, z, logdet, g_scratch_addr[dev], kScratchBytes,
                            (cudaStream_t)stream);
}
