// w4a16_linear_noalloc: the dense W4A16 linear for callers that cannot allocate device memory.
//
// Some callers are handed only their input and output buffers and may not allocate: a plugin or
// custom-op hook inside a host framework that owns every device byte through its own pool (a
// cudaMalloc there escapes the pool's accounting and synchronises the whole device, stalling
// other work), or a runtime that must run inside a fixed, pre-reserved memory budget.  The
// regular w4a16_linear asks them for a workspace (prepared activation rows, split-K partials);
// this entry point takes that scratch from a file-scope device array instead, so nothing is
// allocated per call, and runs the rows in as many chunks as the array needs.
//
// The array is kNoallocScratchBytes (8 MiB) and every GPU that loads the library keeps it until
// the process exits.  Its address is looked up once per device with cudaGetSymbolAddress (the
// array's name is only a host-side stand-in for it); the first call on a device does that set-up,
// so make the first call before any stream capture.  All calls share the array: two calls that
// overlap on the GPU race on it and must be ordered by the caller (one stream, or events).
#include <nvtx3/nvToolsExt.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/w4a16.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;

// Prepared activation rows, then split-K arrival counters and float32 partials.  Zero at module
// load; the counters are cleared again by every call that splits K.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::once_flag g_scratch_once[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices] = {cudaSuccess};

// Device address of the scratch array on the current device (set-up once per device).
void* scratch_for_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) { *err = cudaErrorInvalidDevice; return nullptr; }
  std::call_once(g_scratch_once[dev], [dev]() {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_scratch_ptr[dev] = (g_scratch_err[dev] == cudaSuccess) ? p : nullptr;
  });
  *err = g_scratch_err[dev];
  return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

// from stream_gemm.cu / api.cu (w4_record_status: records the CUDA error behind a W4_ERR_CUDA
// for w4_last_cuda_error, as every other entry point does)
w4_status w4_record_status(w4_status s);
size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count,
                                 bool zp = false);
w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count, uint64_t wait_ns = 0,
                                int stall_after = -1, const uint8_t* zeros = nullptr, int group = 32);

extern "C" {

w4_status w4a16_linear_noalloc(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                               uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
  nvtxRangePushA("w4a16_linear_noalloc");
  struct Pop { ~Pop() { nvtxRangePop(); } } pop;
  if (M < 0 || N < 1 || K < 32 || K % 32 || N > (1LL << 30) || K > (1LL << 30)) return W4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y)) return W4_ERR_INVALID_ARG;
  if (!codes || !scales) return W4_ERR_INVALID_ARG;
  if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3) || (x && !aligned16(x)) ||
      (y && !aligned16(y)))
    return W4_ERR_INVALID_ARG;
  if (M * N > (1LL << 40)) return W4_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return w4_record_status(W4_ERR_CUDA);
  // rows in chunks whose workspace (prepared activation rows, split-K partials) fits the scratch
  auto need_for = [&](int64_t rows) {
    return w4_stream_workspace_bytes(rows, static_cast<int>(N), static_cast<int>(K), 1, W4_EPI_NONE,
                                     true, sms);
  };
  if (M == 0) return W4_OK;
  // The scratch a launch needs is not monotonic in its row count: fewer rows make fewer work
  // units, which can split K and add float32 partials.  So every row count that will actually
  // be launched -- the chunk and the shorter last chunk -- must fit before anything runs.
  if (need_for(1) > kNoallocScratchBytes) return W4_ERR_WORKSPACE;   // one row is too large
  auto fits = [&](int64_t c) {
    const int64_t tail = M % c;
    return need_for(c) <= kNoallocScratchBytes && (tail == 0 || need_for(tail) <= kNoallocScratchBytes);
  };
  int64_t chunk = M;
  while (chunk > 1 && need_for(chunk) > kNoallocScratchBytes) chunk = (chunk + 1) / 2;
  while (chunk > 1 && !fits(chunk)) --chunk;                         // chunk 1 always fits
  cudaError_t err;
  void* ws = scratch_for_current_device(&err);
  if (!ws) return w4_record_status(W4_ERR_CUDA);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int64_t r0 = 0; r0 < M; r0 += chunk) {
    const int64_t rows = M - r0 < chunk ? M - r0 : chunk;
    // (each launch clears the split-K arrival counters it uses)
    const w4_status st = w4_launch_stream_gemm(x + r0 * K, nullptr, 1, codes, scales, nullptr, 1, rows,
                                               static_cast<int>(N), static_cast<int>(K), W4_EPI_NONE,
                                               y + r0 * N, ws, kNoallocScratchBytes, nullptr, s, sms);
    if (st != W4_OK) return w4_record_status(st);
  }
  return W4_OK;
}

}  // extern "C"
