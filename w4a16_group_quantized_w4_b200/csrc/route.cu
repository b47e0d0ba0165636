// Top-k routing, softmax weights and the stable expert-major permutation.
//
// The pages give 128 experts per layer with 8 active per token ("Repacked QAT Gemma 4 26B-A4B
// serves on one TPU v6e at 1.9x FP8 throughput", section "The gap at 26B"); the selection rule
// (largest logits, equal logits by lower index, descending), softmax over the selected, and the
// (expert, pair id) order of the permutation are the definitions stated in w4a16.h.
//
// Mapping:
//   topk     one warp per token.  The lane holding expert e keeps its logits in registers; k rounds
//            of a warp-wide arg-max (value, then lower index) pick the winners.  Lanes 0..k-1 then
//            form the softmax with one exp each and a warp sum.  Per-CTA expert histograms go to
//            the workspace.
//   scatter  every CTA re-derives the global counts and its own base per expert from all CTAs'
//            histograms (deterministic, no atomics on positions), CTA 0 writes expert_offsets,
//            and each warp walks a contiguous run of pairs: a per-warp histogram pass, a scan of
//            the warp bases, then positions from __match_any_sync ranks.  Positions are exact and
//            independent of scheduling.
//   Small T (<= 128) runs in one CTA (one launch) with per-expert token bit masks instead of the
//   scatter (route_fused_kernel); large T uses two launches.
#include "route.cuh"

namespace w4 {

__global__ void __launch_bounds__(kFusedWarps * 32) route_fused_kernel(RouteArgs A) {
  extern __shared__ int smem[];
  route_fused_body<true>(A, smem);
}

__global__ void __launch_bounds__(kRouteWarps * 32) route_topk_kernel(RouteArgs A) {
  extern __shared__ int smem[];
  int* s_cnt = smem;
  pdl_trigger();
  for (int e = threadIdx.x; e < A.E; e += blockDim.x) s_cnt[e] = 0;
  pdl_wait();
  __syncthreads();
  const int t0 = blockIdx.x * A.tokens_per_cta;
  const int t1 = min(A.T, t0 + A.tokens_per_cta);
  topk_dispatch(A, t0, t1, [&](int, int e, int) { atomicAdd(&s_cnt[e], 1); });
  __syncthreads();
  for (int e = threadIdx.x; e < A.E; e += blockDim.x) A.hist[blockIdx.x * A.E + e] = s_cnt[e];
}

__global__ void __launch_bounds__(kRouteWarps * 32) route_scatter_kernel(RouteArgs A) {
  extern __shared__ int smem[];
  int* s_tot = smem;                     // [E]
  int* s_base = s_tot + A.E;             // [E]
  int* s_wcnt = s_base + A.E;            // [nwarps][E]
  const int nctas = gridDim.x;
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e < A.E; e += blockDim.x) {
    int tot = 0, mine = 0;
    for (int c = 0; c < nctas; ++c) {
      const int v = A.hist[c * A.E + e];
      if (c < static_cast<int>(blockIdx.x)) mine += v;
      tot += v;
    }
    s_tot[e] = tot;
    s_base[e] = mine;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < A.E; ++e) {
      const int t = s_tot[e];
      s_tot[e] = run;          // exclusive prefix = expert offset
      run += t;
    }
    if (blockIdx.x == 0) A.expert_offsets[A.E] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < A.E; e += blockDim.x) {
    if (blockIdx.x == 0) A.expert_offsets[e] = s_tot[e];
    s_base[e] += s_tot[e];
  }
  __syncthreads();
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * A.tokens_per_cta * A.k;
  const int64_t p1 = min(static_cast<int64_t>(A.T) * A.k, p0 + static_cast<int64_t>(A.tokens_per_cta) * A.k);
  scatter_pairs(A, p0, p1, s_base, s_wcnt, A.scatter_warps);
}

// ------------------------------------------------------------------------------------------
// combine: y[t] = sum_j w[t, j] * o[pair_pos[t*k + j]], float32 in slot order, bf16 out.
// One thread per 8 consecutive features (16-byte loads and stores); the k row indices and
// weights are fetched first so that the k row loads are in flight together.
// ------------------------------------------------------------------------------------------
template <int KMAX>
__global__ void __launch_bounds__(128) combine_kernel(const uint16_t* __restrict__ o,
                                                      const float* __restrict__ topk_w,
                                                      const int32_t* __restrict__ pair_pos,
                                                      int T, int k, int H, uint16_t* __restrict__ y) {
  const int t = blockIdx.x;
  const int h8 = blockIdx.y * blockDim.x + threadIdx.x;
  pdl_trigger();
  pdl_wait();
  if (t >= T || h8 * 8 >= H) return;
  const int64_t T_k = static_cast<int64_t>(T) * k;
  int64_t row[KMAX];
  float wj[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    row[j] = -1;
    wj[j] = 0.f;
    if (j < k) {
      row[j] = __ldg(pair_pos + static_cast<int64_t>(t) * k + j);
      wj[j] = __ldg(topk_w + static_cast<int64_t>(t) * k + j);
    }
  }
  uint4 v[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    v[j] = make_uint4(0, 0, 0, 0);
    if (j < k && row[j] >= 0 && row[j] < T_k)           // not a valid permutation entry: skip
      v[j] = ldg_stream128(o + row[j] * H + h8 * 8);
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      const uint32_t vv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(wj[j], bf16_lo_to_f32(vv[i]), acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj[j], bf16_hi_to_f32(vv[i]), acc[2 * i + 1]);
      }
    }
  }
  uint4 out;
  out.x = pack_bf16x2(acc[0], acc[1]);
  out.y = pack_bf16x2(acc[2], acc[3]);
  out.z = pack_bf16x2(acc[4], acc[5]);
  out.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(y + static_cast<int64_t>(t) * H + h8 * 8) = out;
}

// ------------------------------------------------------------------------------------------
// chaining of stacked layers: x[t] = bf16(y[t] / sqrt(mean(y[t]^2) + eps)).  One warp per row:
// the lanes' float32 partial sums of squares over 16-byte chunks, combined by a fixed xor tree
// (deterministic), then every element divided by the correctly rounded root (IEEE sqrt and
// division) and rounded to bf16 (nearest even).  The row is read twice (the second time from
// L1 / L2).
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rms_chain_kernel(const uint16_t* __restrict__ y, int64_t T, int H,
                                                        float eps, uint16_t* __restrict__ x) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = H >> 3;
  pdl_trigger();
  pdl_wait();
  for (int64_t t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const uint4* row = reinterpret_cast<const uint4*>(y + t * H);
    float ss = 0.f;
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = __ldg(row + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16_lo_to_f32(w[q]), b = bf16_hi_to_f32(w[q]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(H)) + eps);
    uint4* out = reinterpret_cast<uint4*>(x + t * H);
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = __ldg(row + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o4[q] = pack_bf16x2(__fdiv_rn(bf16_lo_to_f32(w[q]), r), __fdiv_rn(bf16_hi_to_f32(w[q]), r));
      out[i] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
}

}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host launchers (declared in api.cu)
// ---------------------------------------------------------------------------------------------

// The top-k is ALU-bound per SM: spread the tokens over about 128 CTAs, 16 to 64 tokens each.
static int route_tokens_per_cta(int T) {
  int t = (T + 127) / 128;
  return t < w4::kRouteTokensMin ? w4::kRouteTokensMin : (t > w4::kRouteTokensMax ? w4::kRouteTokensMax : t);
}
static int route_num_ctas(int T) { return (T + route_tokens_per_cta(T) - 1) / route_tokens_per_cta(T); }

size_t w4_route_workspace_bytes(int T, int E) {
  if (T <= w4::kFusedMaxT) return 0;   // fused single-CTA path
  return static_cast<size_t>(route_num_ctas(T)) * E * sizeof(int32_t);
}

// Warps taking part in the scatter: (2 + warps) * E ints must stay within 48 KB of shared memory.
static int scatter_warps_for(int E, int max_warps) {
  int w = 12288 / E - 2;
  if (w > max_warps) w = max_warps;
  return w < 1 ? 1 : w;
}

w4_status w4_launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                          int32_t* offsets, int32_t* sorted_pair, int32_t* pair_pos, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  w4::RouteArgs A{logits, T, E, k, ids, w, offsets, sorted_pair, pair_pos, nullptr,
                  route_tokens_per_cta(T), 1};
  const int threads = w4::kRouteWarps * 32;
  // (2 + warps) * E ints <= 40 KB for E <= 1024: within the default shared-memory limit
  if (T == 0) {
    // offsets are all zero
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream) != cudaSuccess) return W4_ERR_CUDA;
    return W4_OK;
  }
  if (w4_route_workspace_bytes(T, E) == 0) {
    // masks [E][ceil(T/32)], offsets [E], ids [T][k], warp sums [32]: <= 36 KB (E <= 1024)
    const size_t smem = (static_cast<size_t>(E) * ((T + 31) / 32) + E + static_cast<size_t>(T) * k + 32) *
                        sizeof(int);
    if (launch_pdl(w4::route_fused_kernel, dim3(1), dim3(w4::kFusedWarps * 32), smem, stream, A) != cudaSuccess)
      return W4_ERR_CUDA;
  } else {
    if (ws == nullptr || ws_bytes < w4_route_workspace_bytes(T, E)) return W4_ERR_WORKSPACE;
    A.hist = static_cast<int32_t*>(ws);
    A.scatter_warps = scatter_warps_for(E, w4::kRouteWarps);
    const size_t smem = static_cast<size_t>(2 + A.scatter_warps) * E * sizeof(int);
    const int nctas = route_num_ctas(T);
    if (launch_pdl(w4::route_topk_kernel, dim3(nctas), dim3(threads), E * sizeof(int), stream, A) != cudaSuccess)
      return W4_ERR_CUDA;
    if (launch_pdl(w4::route_scatter_kernel, dim3(nctas), dim3(threads), smem, stream, A) != cudaSuccess)
      return W4_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_launch_combine(const uint16_t* o, const float* topk_w, const int32_t* pair_pos, int T,
                            int k, int H, uint16_t* y, cudaStream_t stream) {
  if (T == 0) return W4_OK;
  const int threads = 128;
  dim3 grid(T, (H / 8 + threads - 1) / threads);
  cudaError_t e;
  if (k <= 8) e = launch_pdl(w4::combine_kernel<8>, grid, dim3(threads), 0, stream, o, topk_w, pair_pos, T, k, H, y);
  else e = launch_pdl(w4::combine_kernel<32>, grid, dim3(threads), 0, stream, o, topk_w, pair_pos, T, k, H, y);
  if (e != cudaSuccess) return W4_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_launch_rms_chain(const uint16_t* y, int64_t T, int H, float eps, uint16_t* x,
                              cudaStream_t stream, int sm_count) {
  if (T == 0) return W4_OK;
  const int64_t blocks = (T + 7) / 8;
  const int grid = static_cast<int>(blocks < 8LL * sm_count ? blocks : 8LL * sm_count);
  if (launch_pdl(w4::rms_chain_kernel, dim3(grid), dim3(256), 0, stream, y, T, H, eps, x) != cudaSuccess)
    return W4_ERR_CUDA;
  return W4_OK;
}
