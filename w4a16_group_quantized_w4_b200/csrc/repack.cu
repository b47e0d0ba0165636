// Scale recovery ("repack") of bf16 weights that sit on the Q4_0 grid, group 32.
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "A repack, not a re-quantization": a = max|w|; try step a/m for m = 1..8 and keep the first
// that reproduces the group; refine it by least squares; store it at bf16; pack the codes.
// The exact rule (float64, tolerance 1/16, off-grid fallback, zero and non-finite groups) is the
// one stated beside w4_repack in w4a16.h; results are bit-identical to it.
//
// Work mapping: one lane per group (64 input bytes -> 16 code bytes, 2 scale bytes, 1 m byte),
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
  return (i & 1) ? bf16_lo_to_f32(g.v[i >> 1] >> 16) : bf16_lo_to_f32(g.v[i >> 1]);
}

// Bit position of element i's nibble inside code word i / 8 (layout L1: nibble j of a word holds
// element j of its eight, in k order).
__host__ __device__ constexpr int nibble_shift(int i) { return 4 * (i & 7); }

__device__ __forceinline__ int code_of(const uint32_t (&cw)[4], int i) {
  return static_cast<int>((cw[i >> 3] >> nibble_shift(i)) & 15u) - 8;
}

// Exact float64 search and off-grid fallback, the rule's own arithmetic (rarely taken).
__device__ __noinline__ int search_exact(const GroupBits& g, double a, uint32_t (&cw)[4]) {
  for (int m = 1; m <= 8; ++m) {
    const double step = a / static_cast<double>(m);
    bool ok = true;
    uint32_t t[4] = {0, 0, 0, 0};
    for (int i = 0; i < 32; ++i) {
      const double r = static_cast<double>(elem_f32(g, i)) / step;
      const double qi = rint(r);
      if (fabs(r - qi) > 0.0625 || qi < -8.0 || qi > 7.0) { ok = false; break; }
      t[i >> 3] |= static_cast<uint32_t>(static_cast<int>(qi) + 8) << nibble_shift(i);
    }
    if (ok) {
      for (int j = 0; j < 4; ++j) cw[j] = t[j];
      return m;
    }
  }
  const double step8 = a / 8.0;
  uint32_t t[4] = {0, 0, 0, 0};
  for (int i = 0; i < 32; ++i) {
    double qi = rint(static_cast<double>(elem_f32(g, i)) / step8);
    qi = fmin(fmax(qi, -8.0), 7.0);
    t[i >> 3] |= static_cast<uint32_t>(static_cast<int>(qi) + 8) << nibble_shift(i);
  }
  for (int j = 0; j < 4; ++j) cw[j] = t[j];
  return 0;
}

// Work mapping: one lane per group.  The lane holds the group's 64 input bytes (four 16-byte
// loads issued together, and the next group's four issued before this one is decided), so a
// warp decides 32 groups at once and the per-group tail (float64 sum, division, bf16 rounding)
// is shared by 32 groups per warp instruction.
//
// float32 guard-band search over the group (v: element 2j in the low half of v[j]).  Returns m
// in 1..8 (code words in cw, least-squares sums in num / den), or 0 when the exact path must
// decide.  An m for which the smallest nonzero |w| maps to r strictly inside (1/16, 15/16)
// cannot reproduce the group (that element is more than 1/16 from every integer), so it is
// skipped without looking at the elements (margins of 2^-16 cover the float32 error of
// m * wmin / a); on the grid this makes the group's own m the first candidate.  The search runs
// in rounds over the whole warp: each round every undecided group tries its next candidate.
__device__ __forceinline__ int search_fast(const uint32_t (&v)[16], float a, float wmin, float xp,
                                           uint32_t (&cw)[4], double& num, int& den) {
  const float tol = 0.0625f, band = 0x1p-17f, kRound = 12582912.0f;
  const float ra = __frcp_rn(a);
  const float rmin1 = __fmul_rn(wmin, ra);
  auto skip = [&](int m) {
    const float rmin = static_cast<float>(m) * rmin1;
    return rmin > 0.0625f + 0x1p-16f && rmin < 0.9375f - 0x1p-16f;
  };
  int next = 1;
  while (next <= 8 && skip(next)) ++next;
  bool done = next > 8;                      // no candidate at all: off the grid
  int result = 0;
  const unsigned active = __activemask();
  while (__any_sync(active, !done)) {
    const float inv = __fmul_rn(static_cast<float>(next <= 8 ? next : 8), ra);
    uint32_t t[4] = {0u, 0u, 0u, 0u};
    float dmax = 0.f, qs = 0.f;
    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t word = v[i >> 1];
      const float x = (i & 1) ? __uint_as_float(word & 0xFFFF0000u) : __uint_as_float(word << 16);
      const float r = __fmul_rn(x, inv);
      // |r| <= 8 here: adding 1.5 * 2^23 rounds r to an integer n (nearest, ties to even, as
      // rint) and leaves 2^22 + n in the fraction bits, so u = n + 8 is (bits + 8) mod 2^23
      const float tr = __fadd_rn(r, kRound);
      const float qf = __fsub_rn(tr, kRound);
      const uint32_t u = __float_as_uint(tr) + 8u - 0x4B400000u;
      dmax = fmaxf(dmax, fabsf(__fsub_rn(r, qf)));
      t[i >> 3] += u << nibble_shift(i);           // disjoint fields while every u <= 15
      // least-squares sums of this candidate (exact: see the caller)
      ps[i >> 3] = __fmaf_rn(x, qf, ps[i >> 3]);
      qs = __fmaf_rn(qf, qf, qs);
    }
    // u = 16 (n = +8) is the only way out of range.  x -> rint(x * inv) is monotonic, so it
    // happens exactly when it happens for the largest element xp (the same float32 operations)
    const uint32_t up = __float_as_uint(__fadd_rn(__fmul_rn(xp, inv), kRound)) + 8u - 0x4B400000u;
    const bool fail = (dmax > tol + band) || up > 15u;
    const bool unsure = dmax > tol - band;
    if (!done) {
      if (!fail) {
        done = true;
        if (!unsure) {                             // else 0: exact path
          result = next;
#pragma unroll
          for (int j = 0; j < 4; ++j) cw[j] = t[j];
          // On the grid every nonzero product w q lies within a factor 70 of the others and
          // carries at most 12 significant bits, so sums of them are exact in any order: eight
          // in float32 (at most about 21 bits wide), the four partial sums in float64.  This is
          // the float64 index-order sum of the rule, bit for bit.  sum q^2 <= 2048 is exact too.
          num = __dadd_rn(__dadd_rn(static_cast<double>(ps[0]), static_cast<double>(ps[1])),
                          __dadd_rn(static_cast<double>(ps[2]), static_cast<double>(ps[3])));
          den = static_cast<int>(qs);
        }
      } else {
        ++next;
        while (next <= 8 && skip(next)) ++next;
        done = next > 8;                           // off the grid: decided exactly
      }
    }
  }
  return result;
}

// The exact rule (and the off-grid fallback) for one group, with the float64 sum in index order.
// Kept out of line so that the common path's register budget stays small.
__device__ __noinline__ int exact_group(const uint32_t (&v)[16], float a, double& num, int& den,
                                        uint32_t (&cw)[4]) {
  GroupBits G;
#pragma unroll
  for (int j = 0; j < 16; ++j) G.v[j] = v[j];
  uint32_t cws[4] = {0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u};
  const int m = search_exact(G, static_cast<double>(a), cws);
  double nn = 0.0;
  int dd = 0;
  for (int i = 0; i < 32; ++i) {
    const int qi = code_of(cws, i);
    nn = __fma_rn(static_cast<double>(elem_f32(G, i)), static_cast<double>(qi), nn);
    dd += qi * qi;
  }
  num = nn;
  den = dd;
#pragma unroll
  for (int j = 0; j < 4; ++j) cw[j] = cws[j];
  return m;
}

__device__ __forceinline__ void load_group(const uint4* __restrict__ w, int64_t gi, uint4 (&u)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) u[j] = __ldg(w + gi * 4 + j);
}

__global__ void __launch_bounds__(256, 4) repack_kernel(const uint4* __restrict__ w, int64_t groups,
                                                     uint32_t* __restrict__ codes,
                                                     uint16_t* __restrict__ scales,
                                                     uint8_t* __restrict__ group_m,
                                                     unsigned long long* off_grid_count) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint4 nx[4];
  if (gi < groups) load_group(w, gi, nx);
  for (; gi < groups; gi += stride) {
    uint32_t v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[4 * j] = nx[j].x; v[4 * j + 1] = nx[j].y; v[4 * j + 2] = nx[j].z; v[4 * j + 3] = nx[j].w;
    }
    if (gi + stride < groups) load_group(w, gi + stride, nx);   // in flight while this one is decided
    // Largest and smallest nonzero |w| (bf16 magnitude bits), and the largest element, two
    // elements per instruction: |w| - 1 per half-word (zero -> 0xFFFF) is (y + 0x7FFF) ^ 0x8000
    // for y <= 0x7FFF, with no carry between the halves; bf16 bit patterns compared as signed
    // 16-bit integers order the non-negative values (and any non-negative one beats every
    // negative one).
    uint32_t amax2 = 0u, zmin2 = 0xFFFFFFFFu, pmax2 = 0x80008000u;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t y = v[j] & 0x7FFF7FFFu;
      amax2 = __vmaxu2(amax2, y);
      zmin2 = __vminu2(zmin2, (y + 0x7FFF7FFFu) ^ 0x80008000u);
      pmax2 = __vmaxs2(pmax2, v[j]);
    }
    const uint32_t amax = max(amax2 & 0xFFFFu, amax2 >> 16);
    const uint32_t zmin = min(zmin2 & 0xFFFFu, zmin2 >> 16);
    const uint32_t amin = zmin == 0xFFFFu ? 0x7FFFu : zmin + 1u;
    const bool nonfinite = amax >= 0x7F80u;                    // exponent all ones: inf or NaN
    const int16_t p_lo = static_cast<int16_t>(pmax2 & 0xFFFFu), p_hi = static_cast<int16_t>(pmax2 >> 16);
    const uint32_t pbits = static_cast<uint16_t>(p_lo > p_hi ? p_lo : p_hi);
    uint32_t cw[4] = {0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u};   // q = 0
    int m;
    uint16_t scale_bits;
    bool off = false;
    if (nonfinite) {
      m = 0;
      scale_bits = 0x7FC0;
      off = true;
    } else if (amax == 0) {
      m = 1;
      scale_bits = 0;
    } else {
      const float a = bf16_lo_to_f32(amax);
      m = 0;
      double num = 0.0;
      int den = 0;
      if (a >= 0x1p-100f && a <= 0x1p100f)
        m = search_fast(v, a, bf16_lo_to_f32(amin), bf16_lo_to_f32(pbits), cw, num, den);
      if (m == 0) {
        m = exact_group(v, a, num, den, cw);
        off = (m == 0);
      }
      const double s = den > 0 ? __ddiv_rn(num, static_cast<double>(den)) : 0.0;
      scale_bits = f64_to_bf16_rne(s);
    }
    reinterpret_cast<uint4*>(codes)[gi] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    scales[gi] = scale_bits;
    if (group_m) group_m[gi] = static_cast<uint8_t>(m);
    if (off_grid_count) {
      const unsigned active = __activemask();
      const unsigned ballot = __ballot_sync(active, off);
      if (ballot && lane == __ffs(active) - 1)
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
  const int threads = 256;                               // 256 groups per block (one lane each)
  int64_t blocks = (groups + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count) * 16;
  if (blocks > cap) blocks = cap;
  w4::repack_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(w), groups, codes, scales, group_m, off_grid_count);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
