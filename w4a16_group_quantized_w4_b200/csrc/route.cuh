// Routing device code shared by its own kernels (route.cu) and the fused MoE decode kernel
// (fused.cu).  The design notes are at the top of route.cu.
#pragma once

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
static __device__ void scatter_pairs(const RouteArgs& A, int64_t p0, int64_t p1, const int* s_base,
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
// The body (route_fused_kernel, and the routing phase of the fused MoE decode kernel): smem
// holds E * ceil(T / 32) + E + T * k + 32 ints; E <= blockDim.x <= 1024.  PDL: launched with
// programmatic stream serialization (the masks are cleared before waiting for the predecessor).
// FROM_IDS: the top-k is already in topk_ids / topk_w (written earlier in the same kernel by
// route_topk_one); only the offsets and the permutation are formed here.
template <bool PDL, bool FROM_IDS = false>
__device__ __forceinline__ void route_fused_body(const RouteArgs A, int* smem) {
  const int W = (A.T + 31) >> 5;                          // mask words per expert (<= 4)
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem);   // [E][W]
  int* s_off = smem + A.E * W;                            // [E]
  int* s_ids = s_off + A.E;                               // [T][k]
  int* s_wsum = s_ids + A.T * A.k;                        // [32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (PDL) pdl_trigger();
  for (int i = threadIdx.x; i < A.E * W; i += blockDim.x) s_mask[i] = 0u;
  if (PDL) pdl_wait();
  __syncthreads();
  if (FROM_IDS) {
    for (int p = threadIdx.x; p < A.T * A.k; p += blockDim.x) {
      const int t = p / A.k;
      const int e = __ldcg(A.topk_ids + p);
      s_ids[p] = e;
      atomicOr(&s_mask[e * W + (t >> 5)], 1u << (t & 31));
    }
  } else {
    topk_dispatch(A, 0, A.T, [&](int t, int e, int gl) {
      s_ids[t * A.k + gl] = e;
      atomicOr(&s_mask[e * W + (t >> 5)], 1u << (t & 31));
    });
  }
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
    const int v = lane < static_cast<int>(blockDim.x >> 5) ? s_wsum[lane] : 0;
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

// Top-k of one token t by one whole warp (writes topk_ids / topk_w of the token).
__device__ __forceinline__ void route_topk_one(const RouteArgs& A, int t) {
  const int lane = threadIdx.x & 31;
  if (A.E <= 32) topk_token<1, 32>(A, t, 0xffffffffu, lane);
  else if (A.E <= 64) topk_token<2, 32>(A, t, 0xffffffffu, lane);
  else if (A.E <= 128) topk_token<4, 32>(A, t, 0xffffffffu, lane);
  else if (A.E <= 256) topk_token<8, 32>(A, t, 0xffffffffu, lane);
  else if (A.E <= 512) topk_token<16, 32>(A, t, 0xffffffffu, lane);
  else topk_token<32, 32>(A, t, 0xffffffffu, lane);
}

}  // namespace w4
