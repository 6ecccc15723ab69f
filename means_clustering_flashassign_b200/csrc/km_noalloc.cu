// km_noalloc.cu -- km_assign_static: the nearest-centroid assignment for
// callers that cannot allocate device memory.
//
// Some callers own every byte of device memory themselves: a host framework
// that hands out memory only from its own pool (and forbids side
// allocations that would fragment it or break its budget), or a
// latency-critical loop where cudaMalloc's implicit synchronisation and
// unpredictable cost are not acceptable.  They still pass inputs and
// outputs, but cannot provide the scratch workspace km_assign asks for.
//
// This variant takes its scratch from one file-scope device array of fixed
// size instead.  Every GPU that loads libkm.so holds that array until the
// process exits; requests whose scratch would not fit are refused.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/km.h"
#include "km_internal.h"

namespace {

// Scratch size of the static area (16 MiB per device, see km.h).
constexpr size_t kStaticScratchBytes = KM_ASSIGN_STATIC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: host code must obtain the address with
// cudaGetSymbolAddress (below) before handing it to a kernel.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

int static_fail(int code, const char* msg) {
  km::set_last_error(msg);
  return code;
}

// Device address of g_static_scratch on the current device.  Outside stream
// capture it is looked up again on every call (with that device current), so
// a device reset or a re-created context, which reloads the module at a new
// address, is followed.  During capture the address cached by the last
// uncaptured call on the device is used (a lookup may not be legal while a
// capture is open); with no such call the request is refused.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return static_fail(KM_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return static_fail(KM_ERR_UNSUPPORTED, "device ordinal out of range");
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const cudaError_t ce = cudaStreamIsCapturing(stream, &cap);
  if (ce != cudaSuccess) {
    char buf[256];
    snprintf(buf, sizeof(buf), "cudaStreamIsCapturing failed: %s", cudaGetErrorString(ce));
    return static_fail(KM_ERR_CUDA, buf);
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      char buf[256];
      snprintf(buf, sizeof(buf), "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return static_fail(KM_ERR_CUDA, buf);
    }
    g_scratch_addr[dev] = p;
  } else if (!g_scratch_addr[dev]) {
    return static_fail(KM_ERR_UNSUPPORTED,
                       "km_assign_static: the first call on a device must come before any stream capture");
  }
  *out = g_scratch_addr[dev];
  return KM_OK;
}

}  // namespace

extern "C" {

int km_assign_static(const void* X, const void* C, int B, int64_t N, int D, int K, int dtype, int32_t* idx,
                     float* mindist, double* objective, void* stream) {
  km::Plan plan;
  const char* why = "";
  const int pr = km::make_plan(plan, KM_OP_ASSIGN, B, N, D, K, dtype, 0, &why);
  if (pr != KM_OK) return static_fail(pr, why);
  const size_t need = plan.total;
  if (need > kStaticScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "km_assign_static: this shape needs %zu bytes of scratch, the static area holds %zu; "
             "use km_assign with a caller-provided workspace",
             need, kStaticScratchBytes);
    return static_fail(KM_ERR_UNSUPPORTED, buf);
  }
  void* scratch = nullptr;
  const int r = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (r != KM_OK) return r;
  // km_assign clears the status word at the start of the area and fully
  // writes every other scratch value before reading it.
  return km_assign(X, C, B, N, D, K, dtype, idx, mindist, objective, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
