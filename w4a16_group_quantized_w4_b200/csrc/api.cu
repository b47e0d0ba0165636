// C ABI of libw4a16: argument checks, dispatch to the kernels, workspace sizing, status text.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "../../include/w4a16.h"

// A named profiler range around each entry point, so that a timeline (nsys, ncu's NVTX filters)
// shows the library's calls by name; without a profiler attached the calls do nothing.
namespace {
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};
}  // namespace

// kernel launchers (repack.cu, route.cu, stream_gemm.cu)
w4_status w4_launch_repack(const uint16_t* w, int64_t groups, uint32_t* codes, uint16_t* scales,
                           uint8_t* group_m, unsigned long long* off_grid_count,
                           cudaStream_t stream, int sm_count);
size_t w4_route_workspace_bytes(int T, int E);
w4_status w4_launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                          int32_t* offsets, int32_t* sorted_pair, int32_t* pair_pos, void* ws,
                          size_t ws_bytes, cudaStream_t stream);
w4_status w4_launch_combine(const uint16_t* o, const float* topk_w, const int32_t* pair_pos, int T,
                            int k, int H, uint16_t* y, cudaStream_t stream);
w4_status w4_launch_rms_chain(const uint16_t* y, int64_t T, int H, float eps, uint16_t* x,
                              cudaStream_t stream, int sm_count);
size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count,
                                 bool zp = false);
w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count, uint64_t wait_ns = 0,
                                int stall_after = -1, const uint8_t* zeros = nullptr, int group = 32);
size_t w4_tc_workspace_bytes(int64_t rows, int K, int64_t wrows);
size_t w4_layer_workspace_bytes(int T, int E, int k, int H, int I, int sm_count);
size_t w4_layer_control_bytes(int E, int k, int H, int I, int sm_count);
w4_status w4_layer_check(int T, int E, int k, int H, int I);
w4_status w4_launch_moe_layer(const uint16_t* x, const float* logits, int T, int E, int k,
                              const uint32_t* gu_codes, const uint16_t* gu_scales, const uint32_t* dn_codes,
                              const uint16_t* dn_scales, int H, int I, uint16_t* y, void* ws, size_t ws_bytes,
                              int32_t* dev_status, cudaStream_t stream, int sm_count);
bool w4_tm_supported(int N, int K, int epi);
w4_status w4_launch_tm_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                            const uint32_t* codes, const uint16_t* scales, const int32_t* offsets,
                            int E, int64_t rows, int N, int K, int epi, uint16_t* out, void* ws,
                            size_t ws_bytes, int32_t* dev_status, cudaStream_t stream, int sm_count);

// Path choice: the tensor-memory kernel where the routed rows per weight matrix make a real
// dense contraction (on average >= 32 rows per expert, or >= 64 rows for a dense linear) and the
// shapes fit its tiles (weight tiles of 128 rows, K a multiple of 64 up to 4096); the
// weight-streaming kernel otherwise (decode batches, dense GEMVs with split-K over the SMs).
static bool use_tc(int64_t rows, int E, int N, int K, int epi, bool dense, const void* scales) {
  if (!w4_tm_supported(N, K, epi)) return false;
  if (scales && (reinterpret_cast<uintptr_t>(scales) & 3) != 0) return false;
  return dense ? rows >= 64 : rows >= 32LL * E;
}

namespace {

thread_local int32_t g_last_cuda_error = 0;

int current_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

// Returns the status and records the CUDA error behind a W4_ERR_CUDA.
w4_status finish(w4_status s) {
  if (s == W4_ERR_CUDA) {
    cudaError_t e = cudaGetLastError();
    g_last_cuda_error = static_cast<int32_t>(e == cudaSuccess ? cudaErrorUnknown : e);
  }
  return s;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

// Status recording for entry points defined in other files of the library.
w4_status w4_record_status(w4_status s) { return finish(s); }

extern "C" {

const char* w4_status_str(int32_t s) {
  switch (s) {
    case W4_OK: return "W4_OK";
    case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
    case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
    case W4_ERR_CUDA: return "W4_ERR_CUDA";
    case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
    case W4_ERR_WORKSPACE: return "W4_ERR_WORKSPACE";
    default: return "W4_ERR_UNKNOWN";
  }
}

int32_t w4_last_cuda_error(void) { return g_last_cuda_error; }

size_t w4_workspace_bytes(int32_t op, int64_t M_or_T, int64_t N, int64_t K, int32_t E, int32_t k) {
  (void)k;
  if (M_or_T < 0 || N < 0 || K < 0 || E < 0) return 0;
  switch (op) {
    case W4_OP_LINEAR:
      if (N <= 0 || K < 32 || K % 32) return 0;
      if (use_tc(M_or_T, 1, static_cast<int>(N), static_cast<int>(K), W4_EPI_NONE, true, nullptr))
        return w4_tc_workspace_bytes(M_or_T, static_cast<int>(K), N);
      return w4_stream_workspace_bytes(M_or_T, static_cast<int>(N), static_cast<int>(K), 1,
                                       W4_EPI_NONE, true, current_sm_count());
    case W4_OP_ROUTE:
      return w4_route_workspace_bytes(static_cast<int>(M_or_T), E);
    case W4_OP_GMM: {
      // both paths write every routed row once, in pair order, in their own prepared form; the
      // size covers whichever path either epilogue takes
      if (N <= 0 || K < 32 || K % 32 || E < 1 || N > (1LL << 30) || K > (1LL << 30)) return 0;
      size_t need = 0;
      for (int epi : {W4_EPI_NONE, W4_EPI_GELU_GATE}) {
        const size_t b = use_tc(M_or_T, E, static_cast<int>(N), static_cast<int>(K), epi, false, nullptr)
                             ? w4_tc_workspace_bytes(M_or_T, static_cast<int>(K), static_cast<int64_t>(E) * N)
                             : w4_stream_workspace_bytes(M_or_T, static_cast<int>(N), static_cast<int>(K), E,
                                                         epi, false, current_sm_count());
        if (b > need) need = b;
      }
      return need;
    }
    case W4_OP_LINEAR_G:
    case W4_OP_GMM_G:
      // the variants always take the weight-streaming kernel; sized for zero-points (the larger)
      if (N <= 0 || K < 32 || K % 32 || E < 1 || N > (1LL << 30) || K > (1LL << 30)) return 0;
      if (op == W4_OP_LINEAR_G)
        return w4_stream_workspace_bytes(M_or_T, static_cast<int>(N), static_cast<int>(K), 1, W4_EPI_NONE,
                                         true, current_sm_count(), true);
      {
        size_t need = 0;
        for (int epi : {W4_EPI_NONE, W4_EPI_GELU_GATE}) {
          const size_t b = w4_stream_workspace_bytes(M_or_T, static_cast<int>(N), static_cast<int>(K), E, epi,
                                                     false, current_sm_count(), true);
          if (b > need) need = b;
        }
        return need;
      }
    case W4_OP_LAYER:
    case W4_OP_LAYER_CTL:
      if (M_or_T > (1LL << 30) || N > (1LL << 30) || K > (1LL << 30)) return 0;
      if (op == W4_OP_LAYER)
        return w4_layer_workspace_bytes(static_cast<int>(M_or_T), E, k, static_cast<int>(N), static_cast<int>(K),
                                        current_sm_count());
      return w4_layer_control_bytes(E, k, static_cast<int>(N), static_cast<int>(K), current_sm_count());
    default:
      return 0;
  }
}

w4_status w4_repack(const uint16_t* w, int64_t rows, int64_t K, uint32_t* codes, uint16_t* scales,
                    uint8_t* group_m, unsigned long long* off_grid_count, void* stream) {
  const Range range("w4_repack");
  if (rows < 0 || K < 32 || K % 32) return W4_ERR_INVALID_ARG;
  if (rows > 0 && (!w || !codes || !scales)) return W4_ERR_INVALID_ARG;
  if ((w && !aligned(w, 16)) || (codes && !aligned(codes, 16)) || (scales && !aligned(scales, 2)))
    return W4_ERR_INVALID_ARG;
  if (off_grid_count && !aligned(off_grid_count, 8)) return W4_ERR_INVALID_ARG;
  const int64_t groups = rows * (K / 32);
  return finish(w4_launch_repack(w, groups, codes, scales, group_m, off_grid_count,
                                 static_cast<cudaStream_t>(stream), current_sm_count()));
}

w4_status w4a16_linear(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                       uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                       size_t workspace_bytes, void* stream) {
  const Range range("w4a16_linear");
  if (M < 0 || N < 1 || K < 32 || K % 32 || N > (1LL << 30) || K > (1LL << 30)) return W4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y)) return W4_ERR_INVALID_ARG;
  if (!codes || !scales) return W4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || (x && !aligned(x, 16)) || (y && !aligned(y, 16)))
    return W4_ERR_INVALID_ARG;
  if (workspace && !aligned(workspace, 16)) return W4_ERR_INVALID_ARG;
  if (M * N > (1LL << 40)) return W4_ERR_UNSUPPORTED;
  if (use_tc(M, 1, static_cast<int>(N), static_cast<int>(K), W4_EPI_NONE, true, scales) && M < (1LL << 31))
    return finish(w4_launch_tm_gemm(x, nullptr, 1, codes, scales, nullptr, 1, M, static_cast<int>(N),
                                    static_cast<int>(K), W4_EPI_NONE, y, workspace, workspace_bytes,
                                    nullptr, static_cast<cudaStream_t>(stream), current_sm_count()));
  return finish(w4_launch_stream_gemm(x, nullptr, 1, codes, scales, nullptr, 1, M,
                                      static_cast<int>(N), static_cast<int>(K), W4_EPI_NONE, y,
                                      workspace, workspace_bytes, nullptr,
                                      static_cast<cudaStream_t>(stream), current_sm_count()));
}

w4_status moe_route_permute(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* topk_ids,
                            float* topk_w, int32_t* expert_offsets, int32_t* sorted_pair,
                            int32_t* pair_pos, void* workspace, size_t workspace_bytes,
                            void* stream) {
  const Range range("moe_route_permute");
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E) return W4_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * k > (1LL << 30)) return W4_ERR_UNSUPPORTED;
  if (!expert_offsets) return W4_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_pair || !pair_pos)) return W4_ERR_INVALID_ARG;
  return finish(w4_launch_route(logits, T, E, k, topk_ids, topk_w, expert_offsets, sorted_pair,
                                pair_pos, workspace, workspace_bytes,
                                static_cast<cudaStream_t>(stream)));
}

w4_status moe_w4a16_gmm(const uint16_t* a, const int32_t* a_row_of_pair, int32_t k,
                        const uint32_t* codes, const uint16_t* scales, const int32_t* expert_offsets,
                        int32_t E, int64_t rows, int32_t N, int32_t K, int32_t epilogue,
                        uint16_t* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                        void* stream) {
  const Range range("moe_w4a16_gmm");
  if (E < 1 || E > 1024 || rows < 0 || N < 1 || K < 32 || K % 32) return W4_ERR_INVALID_ARG;
  if (epilogue != W4_EPI_NONE && epilogue != W4_EPI_GELU_GATE) return W4_ERR_INVALID_ARG;
  if (epilogue == W4_EPI_GELU_GATE && (N % 2)) return W4_ERR_INVALID_ARG;
  if (a_row_of_pair && k < 1) return W4_ERR_INVALID_ARG;
  if (!codes || !scales || !expert_offsets) return W4_ERR_INVALID_ARG;
  if (rows > 0 && (!a || !out)) return W4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || (a && !aligned(a, 16)) || (out && !aligned(out, 16)))
    return W4_ERR_INVALID_ARG;
  if (static_cast<int64_t>(E) * N > (1LL << 31) - 1 || rows > (1LL << 31) - 1) return W4_ERR_UNSUPPORTED;
  if (use_tc(rows, E, N, K, epilogue, false, scales))
    return finish(w4_launch_tm_gemm(a, a_row_of_pair, k, codes, scales, expert_offsets, E, rows, N, K,
                                    epilogue, out, workspace, workspace_bytes, dev_status,
                                    static_cast<cudaStream_t>(stream), current_sm_count()));
  return finish(w4_launch_stream_gemm(a, a_row_of_pair, k, codes, scales, expert_offsets, E, rows, N,
                                      K, epilogue, out, workspace, workspace_bytes, dev_status,
                                      static_cast<cudaStream_t>(stream), current_sm_count()));
}

// Fault injection for the tests of the bounded waits (not part of the C ABI in w4a16.h): the
// grouped GEMM on the weight-streaming kernel with every wait limited to wait_ns and the producer
// warps stopping after stall_after stages, so that the compute warps' waits run out.  The kernel
// then reports W4_ERR_TIMEOUT in dev_status and returns; nothing faults or hangs.
w4_status w4_testing_stream_gmm_stall(const uint16_t* a, const int32_t* a_row_of_pair, int32_t k,
                                      const uint32_t* codes, const uint16_t* scales,
                                      const int32_t* expert_offsets, int32_t E, int64_t rows, int32_t N,
                                      int32_t K, int32_t epilogue, uint16_t* out, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream,
                                      uint64_t wait_ns, int32_t stall_after) {
  const Range range("w4_testing_stream_gmm_stall");
  if (E < 1 || E > 1024 || rows < 0 || N < 1 || K < 32 || K % 32 || !codes || !scales || !expert_offsets)
    return W4_ERR_INVALID_ARG;
  if (epilogue != W4_EPI_NONE && epilogue != W4_EPI_GELU_GATE) return W4_ERR_INVALID_ARG;
  if (rows > 0 && (!a || !out)) return W4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || (a && !aligned(a, 16)) || (out && !aligned(out, 16)))
    return W4_ERR_INVALID_ARG;
  return finish(w4_launch_stream_gemm(a, a_row_of_pair, k, codes, scales, expert_offsets, E, rows, N,
                                      K, epilogue, out, workspace, workspace_bytes, dev_status,
                                      static_cast<cudaStream_t>(stream), current_sm_count(), wait_ns,
                                      stall_after));
}

static bool group_ok(int64_t group, int64_t K) {
  if (group < 32 || group > K || K % group) return false;
  int64_t g = group / 32;
  return group % 32 == 0 && (g & (g - 1)) == 0;
}

w4_status w4a16_linear_g(const uint16_t* x, const uint32_t* codes, const uint16_t* scales,
                         const uint8_t* zeros, int32_t group, uint16_t* y, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t workspace_bytes, void* stream) {
  const Range range("w4a16_linear_g");
  if (M < 0 || N < 1 || K < 32 || K % 32 || N > (1LL << 30) || K > (1LL << 30)) return W4_ERR_INVALID_ARG;
  if (!group_ok(group, K)) return W4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y)) return W4_ERR_INVALID_ARG;
  if (!codes || !scales) return W4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 2) || (x && !aligned(x, 16)) || (y && !aligned(y, 16)))
    return W4_ERR_INVALID_ARG;
  if (workspace && !aligned(workspace, 16)) return W4_ERR_INVALID_ARG;
  if (M * N > (1LL << 40)) return W4_ERR_UNSUPPORTED;
  return finish(w4_launch_stream_gemm(x, nullptr, 1, codes, scales, nullptr, 1, M, static_cast<int>(N),
                                      static_cast<int>(K), W4_EPI_NONE, y, workspace, workspace_bytes,
                                      nullptr, static_cast<cudaStream_t>(stream), current_sm_count(), 0, -1,
                                      zeros, group));
}

w4_status moe_w4a16_gmm_g(const uint16_t* a, const int32_t* a_row_of_pair, int32_t k,
                          const uint32_t* codes, const uint16_t* scales, const uint8_t* zeros,
                          int32_t group, const int32_t* expert_offsets, int32_t E, int64_t rows,
                          int32_t N, int32_t K, int32_t epilogue, uint16_t* out, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream) {
  const Range range("moe_w4a16_gmm_g");
  if (E < 1 || E > 1024 || rows < 0 || N < 1 || K < 32 || K % 32) return W4_ERR_INVALID_ARG;
  if (!group_ok(group, K)) return W4_ERR_INVALID_ARG;
  if (epilogue != W4_EPI_NONE && epilogue != W4_EPI_GELU_GATE) return W4_ERR_INVALID_ARG;
  if (epilogue == W4_EPI_GELU_GATE && (N % 2)) return W4_ERR_INVALID_ARG;
  if (a_row_of_pair && k < 1) return W4_ERR_INVALID_ARG;
  if (!codes || !scales || !expert_offsets) return W4_ERR_INVALID_ARG;
  if (rows > 0 && (!a || !out)) return W4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 2) || (a && !aligned(a, 16)) || (out && !aligned(out, 16)))
    return W4_ERR_INVALID_ARG;
  if (static_cast<int64_t>(E) * N > (1LL << 31) - 1 || rows > (1LL << 31) - 1) return W4_ERR_UNSUPPORTED;
  return finish(w4_launch_stream_gemm(a, a_row_of_pair, k, codes, scales, expert_offsets, E, rows, N, K,
                                      epilogue, out, workspace, workspace_bytes, dev_status,
                                      static_cast<cudaStream_t>(stream), current_sm_count(), 0, -1, zeros,
                                      group));
}

w4_status moe_w4a16_layer(const uint16_t* x, const float* logits, int32_t T, int32_t E, int32_t k,
                          const uint32_t* gu_codes, const uint16_t* gu_scales, const uint32_t* dn_codes,
                          const uint16_t* dn_scales, int32_t H, int32_t I, uint16_t* y, void* workspace,
                          size_t workspace_bytes, int32_t* dev_status, void* stream) {
  const Range range("moe_w4a16_layer");
  const w4_status chk = w4_layer_check(T, E, k, H, I);
  if (chk != W4_OK) return chk;
  if (T == 0) return W4_OK;
  if (!x || !logits || !gu_codes || !gu_scales || !dn_codes || !dn_scales || !y) return W4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(gu_codes, 16) || !aligned(dn_codes, 16) ||
      !aligned(gu_scales, 4) || !aligned(dn_scales, 4) || (workspace && !aligned(workspace, 256)))
    return W4_ERR_INVALID_ARG;
  return finish(w4_launch_moe_layer(x, logits, T, E, k, gu_codes, gu_scales, dn_codes, dn_scales, H, I, y,
                                    workspace, workspace_bytes, dev_status, static_cast<cudaStream_t>(stream),
                                    current_sm_count()));
}

w4_status moe_combine(const uint16_t* o, const float* topk_w, const int32_t* pair_pos, int32_t T,
                      int32_t k, int32_t H, uint16_t* y, void* stream) {
  const Range range("moe_combine");
  if (T < 0 || k < 1 || H < 8 || H % 8) return W4_ERR_INVALID_ARG;
  if (T > 0 && (!o || !topk_w || !pair_pos || !y)) return W4_ERR_INVALID_ARG;
  if ((o && !aligned(o, 16)) || (y && !aligned(y, 16))) return W4_ERR_INVALID_ARG;
  return finish(w4_launch_combine(o, topk_w, pair_pos, T, k, H, y, static_cast<cudaStream_t>(stream)));
}

w4_status moe_rms_chain(const uint16_t* y, int64_t T, int32_t H, float eps, uint16_t* x_next,
                        void* stream) {
  const Range range("moe_rms_chain");
  if (T < 0 || H < 8 || H % 8 || !(eps >= 0.f) || eps > 1e30f) return W4_ERR_INVALID_ARG;
  if (T > 0 && (!y || !x_next)) return W4_ERR_INVALID_ARG;
  if ((y && !aligned(y, 16)) || (x_next && !aligned(x_next, 16))) return W4_ERR_INVALID_ARG;
  return finish(w4_launch_rms_chain(y, T, H, eps, x_next, static_cast<cudaStream_t>(stream),
                                    current_sm_count()));
}

}  // extern "C"
