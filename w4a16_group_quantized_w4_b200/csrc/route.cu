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
#include "common.cuh"

namespace w4 {

constexpr int kRouteWarps = 8;                 // warps per CTA in the two-launch path
constexpr int kFusedWarps = 32;                // warps of the single-CTA path
constexpr int kRouteTokensMin = 16;            // tokens per CTA in the two-launch path: from 16
constexpr int kRouteTokensMax = 64;            // (top-k spread over many SMs) up to 64 (fewer
                                               // histograms for the scatter to read)
constexpr int kFusedMaxT = 128;                // largest T routed by the single-CTA path

struct RouteArgs {
  const float* logits;
  int T, E, k;
  int32_t* topk_ids;
  float* topk_w;
  int32_t* expert_offsets;
  int32_t* sorted_pair;
  int32_t* pair_pos;
  int32_t* hist;       // [num_ctas][E] per-CTA counts (workspace)
  int tokens_per_cta;
  int scatter_warps;    // warps taking part in the scatter (shared scratch scales with it)
};

// Order-preserving map of a non-NaN float to uint32 (larger value -> larger key); -0 and +0 map
// to the same key, so equal logits compare equal exactly as they do as floats.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of token t by a group of G lanes (a warp, or a half warp with mask gmask); writes
// topk_ids / topk_w and returns, in group lanes 0..k-1, the expert chosen in round `gl` (-1 in
// the other lanes).  PL = logits per lane (E <= G * PL); group lane gl holds experts c * G + gl
// as order keys.  Each round takes the group maximum of the lanes' best untaken keys (one
// redux), then the lowest expert index among the lanes holding it (a second redux).
template <int PL, int G>
__device__ int topk_token(const RouteArgs& A, int t, uint32_t gmask, int gl) {
  uint32_t key[PL];
  const float* row = A.logits + static_cast<int64_t>(t) * A.E;
#pragma unroll
  for (int c = 0; c < PL; ++c) {
    const int e = c * G + gl;
    key[c] = e < A.E ? order_key(__ldg(row + e)) : 0u;     // 0: below every real key
  }
  uint32_t taken = 0;
  uint32_t top = 0, sel_key = 0;
  int sel_e = -1;
  for (int j = 0; j < A.k; ++j) {
    uint32_t bk = 0;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int c = 0; c < PL; ++c) {                    // ascending c: the first maximum is the
      const bool free_c = !((taken >> c) & 1u);         // lowest index of this lane
      if (free_c && key[c] > bk) { bk = key[c]; be = c * G + gl; }
    }
    const uint32_t m = __reduce_max_sync(gmask, bk);
    const int win = static_cast<int>(__reduce_min_sync(gmask, bk == m ? static_cast<uint32_t>(be) : 0x7FFFFFFFu));
    if ((win % G) == gl) taken |= 1u << (win / G);
    if (j == 0) top = m;
    if (gl == j) { sel_key = m; sel_e = win; }
  }
  const float ex = gl < A.k ? expf(key_value(sel_key) - key_value(top)) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(gmask, sum, o);
  if (gl < A.k) {
    A.topk_ids[static_cast<int64_t>(t) * A.k + gl] = sel_e;
    A.topk_w[static_cast<int64_t>(t) * A.k + gl] = ex / sum;
  }
  return sel_e;
}

// Calls f(t, e, gl) for every token t of [t0, t1) after its top-k, with e the expert the group
// lane gl picked (gl < k).  Half warps (two tokens per warp at once) when k <= 16 and E <= 256.
template <int PL, int G, typename F>
__device__ void topk_range(const RouteArgs& A, int t0, int t1, F&& f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  constexpr int kPerWarp = 32 / G;
  const int sub = lane / G, gl = lane % G;
  const uint32_t gmask = G == 32 ? 0xffffffffu : (0xFFFFu << (16 * sub));
  for (int base = t0 + warp * kPerWarp; base < t1; base += nwarps * kPerWarp) {
    const int t = base + sub;
    if (t < t1) {
      const int e = topk_token<PL, G>(A, t, gmask, gl);
      if (gl < A.k) f(t, e, gl);
    }
  }
}

template <typename F>
__device__ void topk_dispatch(const RouteArgs& A, int t0, int t1, F&& f) {
  if (A.k <= 16 && A.E <= 256) {
    if (A.E <= 16) topk_range<1, 16>(A, t0, t1, f);
    else if (A.E <= 32) topk_range<2, 16>(A, t0, t1, f);
    else if (A.E <= 64) topk_range<4, 16>(A, t0, t1, f);
    else if (A.E <= 128) topk_range<8, 16>(A, t0, t1, f);
    else topk_range<16, 16>(A, t0, t1, f);
  } else {
    if (A.E <= 32) topk_range<1, 32>(A, t0, t1, f);
    else if (A.E <= 64) topk_range<2, 32>(A, t0, t1, f);
    else if (A.E <= 128) topk_range<4, 32>(A, t0, t1, f);
    else if (A.E <= 256) topk_range<8, 32>(A, t0, t1, f);
    else if (A.E <= 512) topk_range<16, 32>(A, t0, t1, f);
    else topk_range<32, 32>(A, t0, t1, f);
  }
}

// Positions for pairs [p0, p1) given this CTA's per-expert base s_base[E] (shared).
// s_wcnt: [nwarps][E] shared scratch.
// nwarps warps take part (the others only join the CTA barriers).
__device__ void scatter_pairs(const RouteArgs& A, int64_t p0, int64_t p1, const int* s_base,
                              int* s_wcnt, int nwarps) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool active = warp < nwarps;
  const int64_t n = p1 - p0;
  const int64_t per_warp = (n + nwarps - 1) / nwarps;
  const int64_t w0 = p0 + (active ? warp : nwarps) * per_warp;
  const int64_t w1 = active ? min(p1, w0 + per_warp) : w0;
  int* mycnt = s_wcnt + (active ? warp : 0) * A.E;
  if (active)
    for (int e = lane; e < A.E; e += 32) mycnt[e] = 0;
  __syncwarp();
  for (int64_t p = w0 + lane; p - lane < w1; p += 32) {
    int e = p < w1 ? A.topk_ids[p] : -1;
    if (e >= A.E) e = -1;
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (valid && lane == leader) mycnt[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over warps per expert: base for warp w = s_base[e] + sum_{w' < w} cnt[w'][e]
  for (int e = threadIdx.x; e < A.E; e += blockDim.x) {
    int run = s_base[e];
    for (int w = 0; w < nwarps; ++w) {
      const int c = s_wcnt[w * A.E + e];
      s_wcnt[w * A.E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t p = w0 + lane; p - lane < w1; p += 32) {
    int e = p < w1 ? A.topk_ids[p] : -1;
    if (e >= A.E) e = -1;
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const unsigned lt = peers & ((1u << lane) - 1u);
    if (valid) {
      const int pos = mycnt[e] + __popc(lt);
      if (pos >= 0 && static_cast<int64_t>(pos) < static_cast<int64_t>(A.T) * A.k) {
        A.sorted_pair[pos] = static_cast<int32_t>(p);
        A.pair_pos[p] = pos;
      }
    }
    __syncwarp();
    const int leader = __ffs(peers) - 1;
    if (valid && lane == leader) mycnt[e] += __popc(peers);
    __syncwarp();
  }
}

// One CTA does everything (T <= kFusedMaxT).  A token picks an expert at most once, so the
// tokens routed to expert e form a T-bit mask, and the rank of pair (t, j) among expert e's
// pairs -- ordered by pair id, i.e. by token -- is the number of mask bits below t:
//   offsets     exclusive scan over e of popcount(mask[e])      (one thread per expert)
//   positions   pos(t, j) = offsets[e] + popcount(mask[e] & bits below t)   (one thread per pair)
// Every step is a parallel pass; no serial loop over experts or warps.
__global__ void __launch_bounds__(kFusedWarps * 32) route_fused_kernel(RouteArgs A) {
  extern __shared__ int smem[];
  const int W = (A.T + 31) >> 5;                          // mask words per expert (<= 4)
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem);   // [E][W]
  int* s_off = smem + A.E * W;                            // [E]
  int* s_ids = s_off + A.E;                               // [T][k]
  int* s_wsum = s_ids + A.T * A.k;                        // [32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_trigger();
  for (int i = threadIdx.x; i < A.E * W; i += blockDim.x) s_mask[i] = 0u;
  pdl_wait();
  __syncthreads();
  topk_dispatch(A, 0, A.T, [&](int t, int e, int gl) {
    s_ids[t * A.k + gl] = e;
    atomicOr(&s_mask[e * W + (t >> 5)], 1u << (t & 31));
  });
  __syncthreads();
  // exclusive scan of the per-expert counts (E <= blockDim.x)
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < A.E)
    for (int w = 0; w < W; ++w) cnt += __popc(s_mask[e * W + w]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = s_wsum[lane];
    int wi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    s_wsum[lane] = wi - v;                                // exclusive over warps
  }
  __syncthreads();
  if (e < A.E) {
    const int off = s_wsum[warp] + incl - cnt;
    s_off[e] = off;
    A.expert_offsets[e] = off;
    if (e == A.E - 1) A.expert_offsets[A.E] = off + cnt;
  }
  __syncthreads();
  const int P = A.T * A.k;
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int t = p / A.k;
    const int ex = s_ids[p];
    const uint32_t* m = s_mask + ex * W;
    int rank = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(m[w]);
    const int pos = s_off[ex] + rank;
    A.sorted_pair[pos] = p;
    A.pair_pos[p] = pos;
  }
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
