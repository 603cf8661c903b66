// fdllm_gemm_noalloc: the decoder's tcgen05 GEMM for callers that cannot
// allocate device memory.
//
// The GEMM needs scratch memory when it splits K (float partial tiles, one
// arrival counter per output tile, an error word).  fdllm_gemm takes that
// from a context created with fdllm_create, which allocates.  This entry
// point needs no context: its scratch is the file-scope device array below,
// which every GPU that loads the library holds until the process exits.
//
// Host code must not pass `g_noalloc_scratch` itself to a kernel: in host
// code the name is a host-side shadow, not a device address.  The device
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and cached.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/fdllm.h"
#include "common.cuh"
#include "kernels.h"

namespace fd {
void set_thread_error(const std::string& msg);  // api.cu: fdllm_last_error(NULL)
}

namespace {

// Layout of the scratch array (floats): split-K partial tiles, then the
// per-tile arrival counters, the error word and the self-check words.
constexpr size_t kPartialFloats = (size_t)2 << 20;             // 8 MiB of partial tiles
constexpr int kMaxTiles = 4096;                                 // output tiles (counters)
constexpr size_t kScratchFloats = kPartialFloats + kMaxTiles + 8;

static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceSetup {
  bool ready = false;
  float* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  int num_sms = 0;
};

constexpr int kMaxDevices = 64;
DeviceSetup g_setup[kMaxDevices];
EncodeTiledFn g_encode = nullptr;
std::mutex g_setup_mutex;

int fail(int code, const std::string& msg) {
  fd::set_thread_error("fdllm_gemm_noalloc: " + msg);
  return code;
}

// Once per device, with that device current: the scratch array's device
// address, the SM count, the tensor-map encoder.  No allocation.
int setup_device(int dev, DeviceSetup** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(FDLLM_ERR_ARG, "device index out of range");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceSetup& s = g_setup[dev];
  if (!s.ready) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(FDLLM_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess)
      return fail(FDLLM_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
    if (prop.major != 10) return fail(FDLLM_ERR_ARG, "needs an sm_100 (B200-class) GPU");
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess || !fn)
        return fail(FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    s.scratch = static_cast<float*>(ptr);
    s.num_sms = prop.multiProcessorCount;
    s.ready = true;
  }
  *out = &s;
  return FDLLM_OK;
}

bool encode(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

extern "C" int fdllm_gemm_noalloc(const void* w_dev, const void* x_dev, float* y_dev, int N,
                                  int M, int K, int splits, void* cuda_stream) {
  using namespace fd;
  if (!w_dev || !x_dev || !y_dev || N < 1 || M < 1 || K < 1 || splits < 0)
    return fail(FDLLM_ERR_ARG, "bad GEMM arguments");
  if (K % 64 || ((uintptr_t)w_dev | (uintptr_t)x_dev) % 16)
    return fail(FDLLM_ERR_ARG, "needs K % 64 == 0 and 16-byte aligned w_dev / x_dev");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FDLLM_ERR_CUDA, cudaGetErrorString(e));
  DeviceSetup* ds = nullptr;
  int rc = setup_device(dev, &ds);
  if (rc) return rc;
  const size_t ws_bytes = kPartialFloats * sizeof(float);
  GemmShape gs = plan_gemm_tc(ds->num_sms, N, M, K, true, ws_bytes);
  if (splits > 0) {
    if (splits > gs.kb_total) return fail(FDLLM_ERR_ARG, "more splits than K blocks of 64");
    gs.splits = splits;
    gs.units = gs.n_tiles * gs.n_tt * splits;
    gs.grid = gs.units < ds->num_sms ? gs.units : ds->num_sms;
  }
  // The maximum this entry point accepts: split partials within the 8 MiB
  // of the scratch array, and at most kMaxTiles output tiles.
  if (gs.splits > 1 && (size_t)gs.units * (gs.nt / 2) * 128 > kPartialFloats)
    return fail(FDLLM_ERR_ARG, "split-K partials exceed the 8 MiB scratch array (" +
                                   std::to_string(gs.units) + " units); use fewer splits");
  if (gs.n_tiles * gs.n_tt > kMaxTiles)
    return fail(FDLLM_ERR_ARG, "more than 4096 output tiles (128 features x token tile)");
  CUtensorMap wm, xm;
  const uint64_t x_rows = 2ull * ((M + 31) / 32) * 32;
  if (!encode(&wm, w_dev, N, K, 128) || !encode(&xm, x_dev, x_rows, K, gs.nt))
    return fail(FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  float* scratch = ds->scratch;
  int* counters = reinterpret_cast<int*>(scratch + kPartialFloats);
  int* err = counters + kMaxTiles;
  // counters and the error word must start at zero (a call that stopped on a
  // timeout could leave them set); the partial tiles are overwritten.
  e = cudaMemsetAsync(counters, 0, sizeof(int) * (kMaxTiles + 8), st);
  if (e != cudaSuccess) return fail(FDLLM_ERR_CUDA, cudaGetErrorString(e));
  EpiParams ep{};
  ep.kind = EPI_STORE;
  ep.N = N;
  ep.M = M;
  ep.out = y_dev;
  ep.ld_out = N;
  ep.cap_out = (size_t)M * N;
  ep.check = err + 1;
  GemmScratch sc{scratch, counters, err, kPartialFloats, kMaxTiles};
  e = launch_gemm_tc(&wm, &xm, gs, ep, sc, st);
  if (e != cudaSuccess) return fail(FDLLM_ERR_CUDA, cudaGetErrorString(e));
  int err_host = 0;
  e = cudaMemcpyAsync(&err_host, err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(FDLLM_ERR_CUDA, cudaGetErrorString(e));
  if (err_host & DEV_ERR_TIMEOUT) return fail(FDLLM_ERR_TIMEOUT, "a device-side wait timed out");
  return FDLLM_OK;
}
