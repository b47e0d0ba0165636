// Scale recovery ("repack") of bf16 weights that sit on the Q4_0 grid, group 32.
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "A repack, not a re-quantization": a = max|w|; try step a/m for m = 1..8 and keep the first
// that reproduces the group; refine it by least squares; store it at bf16; pack the codes.
// The exact rule (float64, tolerance 1/16, off-grid fallback, zero and non-finite groups) is the
// one stated beside w4_repack in w4a16.h; results are bit-identical to it.
//
// Work mapping: one thread per group (64 input bytes -> 16 code bytes, 2 scale bytes, 1 m byte),
// grid-stride over all groups.  HBM-bound when the ALU work per group stays small, so the
// m-search runs in float32 with a guard band and only falls back to the exact float64 search
// when the float32 evidence cannot decide:
//   r' = w * (m * rcp(a)) carries three float32 roundings, |r' - r| <= 8 * 3 * 2^-24 < 1.5e-6,
//   while the exact float64 r = w / (a/m) is within 2e-15 of the real quotient.  With a band of
//   delta = 2^-17 (7.6e-6) around the only decision threshold that matters, |r - q| = 1/16,
//   every "certainly passes" / "certainly fails" verdict made on r' is also the verdict on r,
//   and a passing element's rint(r') equals rint(r).  Half-integer ambiguity of rint never
//   matters for passing elements (they sit within 1/16 of an integer) and failing elements fail
//   either way.  a outside [2^-100, 2^100] (reciprocal accuracy) and everything off the grid
//   take the exact path.
#include "common.cuh"

namespace w4 {

// float64 -> bf16 bits, nearest with ties to even, written from the format's definition:
// keep 7 fraction bits (round at bit 45 of the binary64 fraction) for results in bf16's normal
// range, and use the 2^-133 quantum below it.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  const uint16_t sign = static_cast<uint16_t>((b >> 48) & 0x8000u);
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
  if (mag > 0x7FF0000000000000ull) return 0x7FC0;                  // NaN
  if (mag >= 0x47F0000000000000ull) return sign | 0x7F80;          // >= 2^128 or inf
  const int e = static_cast<int>(mag >> 52) - 1023;                // unbiased exponent
  if (e >= -126) {
    const uint64_t lsb = (mag >> 45) & 1ull;
    const uint64_t r = (mag + 0x00000FFFFFFFFFFFull + lsb) >> 45;  // half of the dropped 45 bits, minus 1
    const uint64_t out = r - (static_cast<uint64_t>(1023 - 127) << 7);  // re-bias (carry ok)
    return sign | static_cast<uint16_t>(out >= 0x7F80u ? 0x7F80u : out);
  }
  // |x| < 2^-126: bf16 subnormals are k * 2^-133, k = rint(|x| * 2^133) in 0..128.
  const double k = rint(fabs(x) * 0x1p133);
  return sign | static_cast<uint16_t>(k);
}

struct GroupBits {
  uint32_t v[16];  // 32 bf16 patterns, element 2i in the low half of v[i]
};

__device__ __forceinline__ float elem_f32(const GroupBits& g, int i) {
  return (i & 1) ? bf16_hi_to_f32(g.v[i >> 1]) : bf16_lo_to_f32(g.v[i >> 1]);
}

// Exact float64 search and off-grid fallback, the rule's own arithmetic.
__device__ __forceinline__ int search_exact(const GroupBits& g, double a, int (&q)[32]) {
  for (int m = 1; m <= 8; ++m) {
    const double step = a / static_cast<double>(m);
    bool ok = true;
    for (int i = 0; i < 32; ++i) {
      const double r = static_cast<double>(elem_f32(g, i)) / step;
      const double qi = rint(r);
      if (fabs(r - qi) > 0.0625 || qi < -8.0 || qi > 7.0) { ok = false; break; }
      q[i] = static_cast<int>(qi);
    }
    if (ok) return m;
  }
  const double step8 = a / 8.0;
  for (int i = 0; i < 32; ++i) {
    double qi = rint(static_cast<double>(elem_f32(g, i)) / step8);
    qi = fmin(fmax(qi, -8.0), 7.0);
    q[i] = static_cast<int>(qi);
  }
  return 0;
}

// float32 guard-band search.  Returns m in 1..8 when decided (codes in q), 0 when the exact
// path must decide.
__device__ __forceinline__ int search_fast(const GroupBits& g, float a, int (&q)[32]) {
  const float tol = 0.0625f, band = 0x1p-17f;
  const float ra = __frcp_rn(a);
#pragma unroll 1
  for (int m = 1; m <= 8; ++m) {
    const float inv = __fmul_rn(static_cast<float>(m), ra);
    bool fail = false, unsure = false;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float r = __fmul_rn(elem_f32(g, i), inv);
      const float qf = rintf(r);
      const float d = fabsf(__fsub_rn(r, qf));
      fail |= (d > tol + band) | (qf > 7.0f) | (qf < -8.0f);
      unsure |= (d > tol - band);
      q[i] = static_cast<int>(qf);
    }
    if (fail) continue;
    if (unsure) return 0;
    return m;
  }
  return 0;  // off the grid: decided exactly
}

__global__ void __launch_bounds__(256) repack_kernel(const uint4* __restrict__ w, int64_t groups,
                                                     uint4* __restrict__ codes,
                                                     uint16_t* __restrict__ scales,
                                                     uint8_t* __restrict__ group_m,
                                                     unsigned long long* off_grid_count) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gi < groups;
       gi += stride) {
    GroupBits g;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = ldg_stream128(w + gi * 4 + c);
      g.v[4 * c + 0] = u.x; g.v[4 * c + 1] = u.y; g.v[4 * c + 2] = u.z; g.v[4 * c + 3] = u.w;
    }
    uint32_t amax = 0, nonfinite = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t lo = g.v[i] & 0x7FFFu, hi = (g.v[i] >> 16) & 0x7FFFu;
      amax = max(amax, max(lo, hi));
      nonfinite |= ((lo & 0x7F80u) == 0x7F80u) | ((hi & 0x7F80u) == 0x7F80u);
    }
    int q[32];
    int m;
    uint16_t scale_bits;
    bool off = false;
    if (nonfinite) {
#pragma unroll
      for (int i = 0; i < 32; ++i) q[i] = 0;
      m = 0;
      scale_bits = 0x7FC0;
      off = true;
    } else if (amax == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) q[i] = 0;
      m = 1;
      scale_bits = 0;
    } else {
      const float a = bf16_lo_to_f32(amax);
      m = 0;
      if (a >= 0x1p-100f && a <= 0x1p100f) m = search_fast(g, a, q);
      if (m == 0) m = search_exact(g, static_cast<double>(a), q);
      off = (m == 0);
      // least squares with the codes fixed: s* = sum w q / sum q^2, index order, float64
      double num = 0.0;
      int den = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        num = __dadd_rn(num, __dmul_rn(static_cast<double>(elem_f32(g, i)), static_cast<double>(q[i])));
        den += q[i] * q[i];
      }
      const double s = den > 0 ? __ddiv_rn(num, static_cast<double>(den)) : 0.0;
      scale_bits = f64_to_bf16_rne(s);
    }
    uint4 packed;
    uint32_t* pw = reinterpret_cast<uint32_t*>(&packed);
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)   // even elements in the low half-word, odd in the high
        word |= static_cast<uint32_t>(q[8 * wd + j] + 8) << (4 * (j >> 1) + 16 * (j & 1));
      pw[wd] = word;
    }
    codes[gi] = packed;
    scales[gi] = scale_bits;
    if (group_m) group_m[gi] = static_cast<uint8_t>(m);
    if (off_grid_count) {
      const unsigned ballot = __ballot_sync(__activemask(), off);
      const int lane = threadIdx.x & 31;
      if (ballot && lane == __ffs(__activemask()) - 1)
        atomicAdd(off_grid_count, static_cast<unsigned long long>(__popc(ballot)));
    }
  }
}

}  // namespace w4

// Host launcher (declared in api.cu).
w4_status w4_launch_repack(const uint16_t* w, int64_t groups, uint32_t* codes, uint16_t* scales,
                           uint8_t* group_m, unsigned long long* off_grid_count,
                           cudaStream_t stream, int sm_count) {
  if (off_grid_count) {
    if (cudaMemsetAsync(off_grid_count, 0, sizeof(unsigned long long), stream) != cudaSuccess)
      return W4_ERR_CUDA;
  }
  if (groups == 0) return W4_OK;
  const int threads = 256;
  int64_t blocks = (groups + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count) * 8;
  if (blocks > cap) blocks = cap;
  w4::repack_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(w), groups, reinterpret_cast<uint4*>(codes), scales, group_m,
      off_grid_count);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
