// Device half of the seeded input generators (libw4synth.so): the planted bf16 weights of the
// repack workload, drawn group by group with the same counter-based SplitMix64 recipe as
// synth.planted_groups, so that any group's values are identical on the host and the device.
// This is input generation for tests and benchmarks, not part of the W4A16 method: nothing here
// searches, refines or packs scales.
//
// Recipe per group (global index gi) and attempt a = 0..15, counters base = (gi * 16 + a) * 64:
//   p     = 1 + below(draw(base + 32), 8)                   peak level
//   s     = 0x38D2 + below(draw(base + 33), 0x3DCD - 0x38D2 + 1)   bf16 scale pattern
//   pos   = below(draw(base + 34), 32), neg = top bit of draw(base + 35)
//   q[j]  = -p + below(draw(base + j), min(p, 7) + p + 1), j = 0..31
//   q[pos] = -8 if p == 8 else (neg ? -p : p)
// a group whose |q| share a factor > 1 is redrawn with the next attempt; after the last one the
// element after the peak is set to 1.  w = bf16_rne(float(s) * q) (the product is exact in fp32).
// draw(c) = splitmix64(key + c), key = splitmix64(seed << 16 + stream), below(r, n) = ((r >> 32) * n) >> 32.
#include <cuda_runtime.h>

#include <cstdint>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kMix1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t kMix2 = 0x94D049BB133111EBull;
constexpr int kAttempts = 16;
constexpr int kSlots = 64;
constexpr uint32_t kScaleLo = 0x38D2, kScaleHi = 0x3DCD;

__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + kGamma;
  z = (z ^ (z >> 30)) * kMix1;
  z = (z ^ (z >> 27)) * kMix2;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint32_t below(uint64_t r, uint32_t n) {
  return static_cast<uint32_t>(((r >> 32) * static_cast<uint64_t>(n)) >> 32);
}

__device__ __forceinline__ int gcd_small(int a, int b) {
  while (b) { const int t = a % b; a = b; b = t; }
  return a;
}

struct Group {
  int q[32];
  uint32_t s;
  int p;
};

__device__ void draw_group(uint64_t key, uint64_t gi, Group& G) {
  for (int a = 0; a < kAttempts; ++a) {
    const uint64_t base = (gi * kAttempts + a) * kSlots;
    const int p = 1 + static_cast<int>(below(splitmix64(key + base + 32), 8));
    const uint32_t s = kScaleLo + below(splitmix64(key + base + 33), kScaleHi - kScaleLo + 1);
    const int pos = static_cast<int>(below(splitmix64(key + base + 34), 32));
    const bool neg = (splitmix64(key + base + 35) >> 63) != 0;
    const int lo = -p, hi = p < 7 ? p : 7;
    int g = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      int v = lo + static_cast<int>(below(splitmix64(key + base + j), static_cast<uint32_t>(hi - lo + 1)));
      if (j == pos) v = p == 8 ? -8 : (neg ? -p : p);
      G.q[j] = v;
      g = gcd_small(g, v < 0 ? -v : v);
    }
    G.s = s;
    G.p = p;
    if (g == 1) return;
    if (a == kAttempts - 1) {
      const int nxt = (pos + 1) & 31;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j == nxt) G.q[j] = 1;
      return;
    }
  }
}

// bf16 round to nearest even of a finite float32 bit pattern (integer arithmetic)
__device__ __forceinline__ uint16_t f32_bits_to_bf16(uint32_t b) {
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__global__ void planted_kernel(uint64_t key, int64_t group0, int64_t ngroups, uint16_t* w,
                               int8_t* q_out, uint16_t* s_out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < ngroups;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    Group G;
    draw_group(key, static_cast<uint64_t>(group0 + i), G);
    const float sf = __uint_as_float(G.s << 16);
    uint32_t packed[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const uint16_t lo = f32_bits_to_bf16(__float_as_uint(sf * static_cast<float>(G.q[j])));
      const uint16_t hi = f32_bits_to_bf16(__float_as_uint(sf * static_cast<float>(G.q[j + 1])));
      packed[j / 2] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(w + i * 32);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    if (q_out) {
      uint32_t qq[8];
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        qq[j / 4] = (static_cast<uint32_t>(G.q[j] & 0xFF)) | (static_cast<uint32_t>(G.q[j + 1] & 0xFF) << 8) |
                    (static_cast<uint32_t>(G.q[j + 2] & 0xFF) << 16) | (static_cast<uint32_t>(G.q[j + 3] & 0xFF) << 24);
      uint4* qd = reinterpret_cast<uint4*>(q_out + i * 32);
      qd[0] = make_uint4(qq[0], qq[1], qq[2], qq[3]);
      qd[1] = make_uint4(qq[4], qq[5], qq[6], qq[7]);
    }
    if (s_out) s_out[i] = static_cast<uint16_t>(G.s);
  }
}

// Groups whose packed codes (4 words per group, layout L1: in word t, bits 4j..4j+3 hold u = q + 8
// of element 8t + j) differ from the planted codes.
__global__ void mismatch_kernel(uint64_t key, int64_t group0, int64_t ngroups, const uint32_t* codes,
                                unsigned long long* count) {
  unsigned long long bad = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < ngroups;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    Group G;
    draw_group(key, static_cast<uint64_t>(group0 + i), G);
    const uint4 c = *reinterpret_cast<const uint4*>(codes + i * 4);
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    bool same = true;
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int j = 0; j < 8; ++j) same &= static_cast<int>((cw[t] >> (4 * j)) & 15u) - 8 == G.q[8 * t + j];
    bad += same ? 0 : 1;
  }
  for (int o = 16; o; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(count, bad);
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = (n + 255) / 256;
  return static_cast<int>(blocks < 8LL * sms ? (blocks > 0 ? blocks : 1) : 8LL * sms);
}

}  // namespace

extern "C" {

// Planted groups group0 .. group0 + ngroups - 1 of (seed, stream): w [ngroups, 32] bf16 bits
// (16-byte aligned), optionally the planted codes q [ngroups, 32] int8 and scales s [ngroups].
// Returns a cudaError_t value (0 on success).
int w4s_planted(uint64_t seed, uint32_t stream, int64_t group0, int64_t ngroups, uint16_t* w,
                int8_t* q, uint16_t* s, void* cuda_stream) {
  if (ngroups <= 0) return 0;
  const uint64_t key = splitmix64((seed << 16) + stream);
  planted_kernel<<<grid_for(ngroups), 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      key, group0, ngroups, w, q, s);
  return static_cast<int>(cudaGetLastError());
}

// Adds to *count (device) the number of groups among group0 .. group0 + ngroups - 1 whose packed
// codes (ngroups * 4 words) are not the planted ones.
int w4s_code_mismatches(uint64_t seed, uint32_t stream, int64_t group0, int64_t ngroups,
                        const uint32_t* codes, unsigned long long* count, void* cuda_stream) {
  if (ngroups <= 0) return 0;
  const uint64_t key = splitmix64((seed << 16) + stream);
  mismatch_kernel<<<grid_for(ngroups), 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      key, group0, ngroups, codes, count);
  return static_cast<int>(cudaGetLastError());
}

}  // extern "C"
