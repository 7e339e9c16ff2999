// bsa_select_noalloc: the selection call for callers that cannot allocate
// device memory. Its workspace is a fixed array in device memory that the
// library itself defines; the work is done by the ordinary bsa_select path.
//
// Why: some callers may not call cudaMalloc at all once they are running --
// for example a plugin inside a host process that owns all device memory
// through its own pool (a direct cudaMalloc would bypass that pool's budget and
// accounting), or a latency-critical serving loop where a cudaMalloc could
// synchronise the device. Such a caller passes inputs and outputs only.
//
// The array is kSelectScratchBytes (32 MiB). Every GPU that loads libbsa.so
// keeps that much memory reserved until the process exits. All calls share it:
// two calls whose work overlaps on the GPU (different streams, or different
// host threads on one device) race on it and give wrong results, so the caller
// must order them. Nothing in it has to start at zero (the selection kernels
// write every scratch entry they later read), and it keeps whatever the last
// call left there.
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kSelectScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_select_scratch[kSelectScratchBytes];

// Device address of g_select_scratch in the current device's current context. In host
// code the name g_select_scratch is only a host-side stand-in for the symbol, never a
// device address, so the address is looked up with the device current. It is looked up
// on every call (a host-side table lookup once the module is loaded): an address cached
// across calls could go stale after cudaDeviceReset, or belong to another context made
// current on the same device.
bsa_status scratch_for_current_device(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
  if (e != cudaSuccess || !p) {
    bsa::set_last_error("bsa_select_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    return BSA_ERR_CUDA;
  }
  *out = p;
  return BSA_OK;
}

}  // namespace

extern "C" size_t bsa_select_noalloc_max_bytes(void) { return kSelectScratchBytes; }

extern "C" bsa_status bsa_select_noalloc(const bsa_shape* shape, const bsa_select_params* params,
                                         const float* scores, int32_t* kv_idx, int32_t* kv_cnt,
                                         float* sigma, float* sigma_bar, uint8_t* trigger,
                                         float* theta, int32_t* dev_status, void* stream) {
  const size_t need = bsa_select_workspace_bytes(shape, params);
  if (need == 0) {
    // invalid shape or parameters: let the ordinary path report the reason
    return bsa_select(shape, params, scores, kv_idx, kv_cnt, sigma, sigma_bar, trigger, theta,
                      dev_status, nullptr, 0, stream);
  }
  if (need > kSelectScratchBytes) {
    bsa::set_last_error(
        "bsa_select_noalloc: this shape needs %zu bytes of scratch, above the %zu-byte static "
        "maximum; use bsa_select with a caller-provided workspace",
        need, kSelectScratchBytes);
    return BSA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  bsa_status st = scratch_for_current_device(&ws);
  if (st != BSA_OK) return st;
  return bsa_select(shape, params, scores, kv_idx, kv_cnt, sigma, sigma_bar, trigger, theta,
                    dev_status, ws, kSelectScratchBytes, stream);
}
