// Tensor-core (tcgen05 / TMEM) W4A16 grouped GEMM for many tokens per weight matrix (prefill).
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "What changed in vLLM's TPU backend": the grouped matmul takes a scale per 32-wide group and
// dequantises each weight tile in fast on-chip memory before the multiply; activations stay bf16.
// Here the dequantised tile lives in shared memory as the operand of tcgen05.mma, in fp16 rather
// than bf16: s * q has at most 11 significant bits (8 from the bf16 scale, 3 from |q| <= 8), which
// fp16 holds exactly and bf16 does not, so every product the tensor core forms is the exact
// a * (s * q) and only the fp32 accumulation and the output rounding remain.  Range is handled by
// powers of two: each activation row is converted once to fp16(a * 2^f) with f chosen from the
// row's largest magnitude (a_to_f16_kernel), each weight row of a tile uses scales s * 2^e with e
// chosen from the row's largest scale, and the epilogue multiplies by 2^-f and 2^-e, both exact.
//
// Tile: 128 routed rows (M, tokens) x 128 weight rows (N) with K in chunks of 64, accumulated in
// fp32 in tensor memory.  D = A * B^T with A = activations [128 x K] and B = dequantised weights
// [128 x K], both K-major with the 128-byte swizzle (8-row atoms of 1024 bytes, 16-byte chunk c of
// row r stored at chunk c ^ (r % 8)).  With the GELU gate the 128 weight rows are 64 gate rows and
// the 64 up rows of the same outputs, so one thread's accumulator row holds both.
//
// Roles (persistent CTA, one per SM, 16 warps):
//   warp 0       producer: per chunk, the 128 converted activation rows (a 2-D TMA tile; gathered
//                rows were put in pair order by the conversion) into the swizzled A stage and the
//                raw codes of the 128 weight rows by 2-D TMA
//   warp 1       TMEM allocation and the single MMA-issuing thread
//   warp 2       per tile, the tile's scale block by cp.async into bank-padded rows
//   warps 4-7    epilogue: tcgen05.ld of the accumulator, GELU gate / bf16, global stores
//   warps 8-15   dequant: codes + scales -> fp16(s * 2^e * q) into the swizzled B stage
// Every wait is bounded (W4_ERR_TIMEOUT in dev_status instead of a hang).
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"

namespace w4 {
namespace tc {

constexpr int kBM = 128;               // routed rows per tile (MMA M)
constexpr int kBN = 128;               // weight rows per tile (MMA N)
constexpr int kBK = 64;                // k per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 16 * 32;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB
constexpr int kBBytes = kBN * kBK * 2;          // 16 KB
constexpr int kRawBytes = kBN * kBK / 2;        // 4 KB of packed codes
constexpr int kMaxKg = 128;                     // K <= 4096 on this path
// Per-tile scale block: 128 weight rows x kg/2 words (two groups a word), rows padded to an odd
// number of words so that 32 threads reading 32 consecutive rows hit 32 different banks.
constexpr int kScaleBytes = kBN * (kMaxKg / 2 + 1) * 4;   // per buffer (two buffers)
constexpr uint32_t kTmemCols = 256;             // two fp32 accumulators of 128 columns
constexpr int kShRing = 2;                      // per-tile weight-row multipliers 2^-e

struct TcArgs {
  const float* rowmul;      // [rows] 2^-f of each converted activation row
  const uint16_t* scales;
  const int32_t* offsets;   // [E+1] or null (dense: one expert with `rows` rows)
  int E, N, K, kg;
  int64_t rows;
  int epi;
  uint16_t* out;
  int n_tiles;
  int32_t* dev_status;
};

struct Smem {
  static constexpr int a = 0;                                  // kStages x 16 KB (1024-aligned)
  static constexpr int b = a + kStages * kABytes;              // kStages x 16 KB
  static constexpr int raw = b + kStages * kBBytes;            // kStages x 4 KB
  static constexpr int sc = raw + kStages * kRawBytes;         // 2 x 32 KB
  static constexpr int bars = sc + 2 * kScaleBytes;
  // barriers: a_full, raw_full, b_full, raw_empty, ab_empty (x kStages), acc_full, acc_empty,
  // sc_full, sc_empty (x 2), sh_full, sh_empty (x kShRing)
  static constexpr int nbars = 5 * kStages + 8 + 2 * kShRing;
  static constexpr int tmem_slot = bars + nbars * 8;
  static constexpr int sh = tmem_slot + 16;                    // float [kShRing][kBN]
  static constexpr int table = sh + kShRing * kBN * 4;         // int table[E+1], offs[E+1]
};

struct Tile {
  int e, mt, nt;
  int64_t r0;
  int mrows;
};

__device__ __forceinline__ void decode_tile(const TcArgs& A, const int* table, const int* offs,
                                            int t, Tile& T) {
  int lo = 0, hi = A.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (table[mid] <= t) lo = mid; else hi = mid - 1;
  }
  T.e = lo;
  const int off0 = offs[lo], off1 = offs[lo + 1];
  const int nm = (off1 - off0 + kBM - 1) / kBM;
  const int local = t - table[lo];
  T.nt = local / nm;                 // m-tiles fastest: CTAs running together share the weights
  T.mt = local - T.nt * nm;
  T.r0 = off0 + T.mt * kBM;
  T.mrows = min(kBM, off1 - static_cast<int>(T.r0));
}

// global weight row of tile row r (0..127)
__device__ __forceinline__ int64_t wrow(const TcArgs& A, const Tile& T, int r) {
  int n;
  if (A.epi == W4_EPI_GELU_GATE) {
    const int j = T.nt * (kBN / 2) + (r & (kBN / 2 - 1));
    n = (r < kBN / 2) ? j : (A.N >> 1) + j;
  } else {
    n = T.nt * kBN + r;
  }
  return static_cast<int64_t>(T.e) * A.N + n;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: start address, stride
// between 8-row atoms 1024 bytes, descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;                 // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                 // version
  d |= static_cast<uint64_t>(2) << 61;                 // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B (format code 0), both
// K-major, N and M.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) |                                   // D format fp32
         (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 4-bit fields u (bits 0-3 and 16-19 of v) -> the fp16 pair (u - 8): 0x6400 | u is the fp16
// value 1024 + u, and subtracting 1032 is exact.
__device__ __forceinline__ uint32_t nibbles_to_f16x2(uint32_t v) {
  uint32_t r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(0x000F000Fu), "r"(0x64006400u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(r), "r"(0x64086408u));
  return q;
}
__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }   // |e| <= 126

// Power-of-two exponent that brings a finite magnitude with bf16 bit pattern m (sign cleared) to
// [2^(top), 2^(top+1)); 0 for m == 0.  Clamped to +-100 so that 2^e and 2^-e stay normal floats.
__device__ __forceinline__ int shift_for(uint32_t m, int top) {
  if (m == 0) return 0;
  int E = static_cast<int>(m >> 7);
  if (E == 0) E = 1;                                   // subnormal: below 2^-126
  int e = top + 127 - E;
  return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// One warp per output row p: the activation row it reads (row p of `a`, or row
// a_row_of_pair[p] / k_div when rows are gathered) is scanned for its largest finite |a|, which
// picks f so that it lands in [2^14, 2^15); row p of a16 becomes fp16(a * 2^f) and rowmul[p] = 2^-f.
// A bf16 value of magnitude at least 2^-17 is a multiple of 2^-24 with 8 significant bits, so fp16
// holds it exactly: every element within a factor 2^31 of the row's largest converts exactly,
// smaller ones round to the fp16 subnormal grid.  Infinities and NaNs pass through as fp16 inf /
// NaN.  Writing the gathered rows in pair order lets the GEMM read whole 128-row tiles by TMA.
__global__ void __launch_bounds__(256)
a_to_f16_kernel(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair, int k_div,
                int64_t a_rows, int64_t rows, int K, uint16_t* __restrict__ a16,
                float* __restrict__ rowmul, int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = K >> 3;
  for (int64_t row = blockIdx.x * wpb + (threadIdx.x >> 5); row < rows; row += gridDim.x * wpb) {
    int64_t srow = row;
    if (a_row_of_pair) {
      srow = __ldg(a_row_of_pair + row) / k_div;
      if (srow < 0 || srow >= a_rows) {
        if (lane == 0) set_status(dev_status, W4_ERR_INVALID_ARG);
        srow = 0;
      }
    }
    const uint4* src = reinterpret_cast<const uint4*>(a + srow * K);
    uint32_t m = 0;
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
        if (lo < 0x7F80u) m = max(m, lo);
        if (hi < 0x7F80u) m = max(m, hi);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int f = shift_for(m, 14);
    const float mul = pow2f(f);
    uint4* dst = reinterpret_cast<uint4*>(a16 + row * K);
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h = __floats2half2_rn(bf16_lo_to_f32(w[j]) * mul, bf16_hi_to_f32(w[j]) * mul);
        o[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
      dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (lane == 0) rowmul[row] = pow2f(-f);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
               const __grid_constant__ CUtensorMap tmap_a, TcArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint64_t* a_full = bars;
  uint64_t* raw_full = bars + kStages;
  uint64_t* b_full = bars + 2 * kStages;
  uint64_t* raw_empty = bars + 3 * kStages;
  uint64_t* ab_empty = bars + 4 * kStages;
  uint64_t* acc_full = bars + 5 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* sc_full = acc_full + 4;
  uint64_t* sc_empty = acc_full + 6;
  uint64_t* sh_full = acc_full + 8;
  uint64_t* sh_empty = sh_full + kShRing;
  float* sh = reinterpret_cast<float*>(smem + Smem::sh);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::tmem_slot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::tmem_slot + 8);
  int* table = reinterpret_cast<int*>(smem + Smem::table);
  int* offs = table + (A.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile table (same validation as the streaming kernel)
  if (warp == 0) {
    int run = 0;
    bool bad = false;
    if (A.offsets && lane == 0) bad = (A.offsets[0] != 0) || (A.offsets[A.E] != A.rows);
    for (int base = 0; base < A.E; base += 32) {
      const int e = base + lane;
      int cnt = 0;
      if (e < A.E) {
        const int64_t o0 = A.offsets ? A.offsets[e] : 0;
        const int64_t o1 = A.offsets ? A.offsets[e + 1] : A.rows;
        if (o1 < o0 || o0 < 0 || o1 > A.rows) bad = true;
        cnt = o1 > o0 ? static_cast<int>((o1 - o0 + kBM - 1) / kBM) * A.n_tiles : 0;
        offs[e] = static_cast<int>(o0);
        if (e == A.E - 1) offs[A.E] = static_cast<int>(o1);
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < A.E) table[e] = run + incl - cnt;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) table[A.E] = bad ? 0 : run;
    if (bad && lane == 0) set_status(A.dev_status, W4_ERR_INVALID_ARG);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&a_full[s], 1);      // expect_tx by the producer's lane 0
      mbar_init(&raw_full[s], 1);
      mbar_init(&b_full[s], 8);      // one arrival per dequant warp
      mbar_init(&raw_empty[s], 8);
      mbar_init(&ab_empty[s], 1);    // tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);   // one arrival per epilogue warp
      mbar_init(&sc_full[b], 32);    // the scale loader's lanes (cp.async arrivals)
      mbar_init(&sc_empty[b], 8);
    }
    for (int b = 0; b < kShRing; ++b) {
      mbar_init(&sh_full[b], 4);     // the four dequant warps of the first k half
      mbar_init(&sh_empty[b], 4);    // the four epilogue warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = table[A.E];
  const int nk = (A.K + kBK - 1) / kBK;

  auto fail = [&](int lane_id) {
    if (lane_id == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); *abort_flag = 1; }
  };

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) prefetch_tmap(&tmap_codes);
    int slot = 0;
    uint32_t ph = 0;
    bool lap0 = true;
    int ti = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++ti) {
      Tile T;
      decode_tile(A, table, offs, t, T);
      const int64_t row_a = wrow(A, T, 0), row_b = wrow(A, T, kBN / 2);
      for (int kc = 0; kc < nk; ++kc) {
        if (!lap0) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&ab_empty[slot], ph) && mbar_wait(&raw_empty[slot], ph);
          if (!__shfl_sync(0xffffffffu, ok, 0)) { fail(lane); return; }
        }
        uint8_t* adst = smem + Smem::a + slot * kABytes;
        uint8_t* rdst = smem + Smem::raw + slot * kRawBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[slot], kRawBytes);
          tma_load_2d(rdst, &tmap_codes, kc * 8, static_cast<int32_t>(row_a), &raw_full[slot]);
          tma_load_2d(rdst + (kBN / 2) * 32, &tmap_codes, kc * 8, static_cast<int32_t>(row_b),
                      &raw_full[slot]);
          mbar_arrive_expect_tx(&a_full[slot], kABytes);
          tma_load_2d(adst, &tmap_a, kc * kBK, static_cast<int32_t>(T.r0), &a_full[slot]);
        }
        if (++slot == kStages) { slot = 0; if (!lap0) ph ^= 1u; lap0 = false; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kBM, kBN);
      int slot = 0;
      uint32_t ph = 0;
      int ti = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
        const int ab = ti & 1;
        if (ti >= 2 && !mbar_wait(&acc_empty[ab], ((ti >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kBN;
        for (int kc = 0; kc < nk; ++kc) {
          if (!mbar_wait(&a_full[slot], ph) || !mbar_wait(&b_full[slot], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + Smem::a + slot * kABytes);
          const uint32_t b_base = smem_u32(smem + Smem::b + slot * kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            mma_f16(d_tmem, sw128_desc(a_base + k * 32), sw128_desc(b_base + k * 32), idesc,
                     (kc | k) != 0 ? 1u : 0u);
          }
          mma_commit(&ab_empty[slot]);   // frees the A / B stage once these MMAs have read it
          if (++slot == kStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);       // accumulator ready once every MMA of the tile is done
      }
      if (!ok) fail(0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------ scale loader ------------------------------
    const int hw = A.kg >> 1;                 // words per row in global memory
    const int P = hw | 1;                     // words per row in shared memory (odd)
    int ti = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++ti) {
      Tile T;
      decode_tile(A, table, offs, t, T);
      const int sb = ti & 1;
      if (ti >= 2 && !mbar_wait(&sc_empty[sb], ((ti >> 1) - 1) & 1)) { fail(lane); break; }
      const uint32_t dst0 = smem_u32(smem + Smem::sc + sb * kScaleBytes);
      const uint32_t* src_a = reinterpret_cast<const uint32_t*>(A.scales + wrow(A, T, 0) * A.kg);
      const uint32_t* src_b = reinterpret_cast<const uint32_t*>(A.scales + wrow(A, T, kBN / 2) * A.kg);
      for (int w = lane; w < kBN * hw; w += 32) {
        const int rr = w / hw, j = w - rr * hw;
        const uint32_t* src = rr < kBN / 2 ? src_a + w : src_b + (w - (kBN / 2) * hw);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                     ::"r"(dst0 + (rr * P + j) * 4), "l"(src) : "memory");
      }
      // each lane's arrival lands once its copies have
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sc_full[sb]))
                   : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------ epilogue ------------------------------
    const int q = warp - 4;             // TMEM lanes 32q .. 32q + 31
    const int row = q * 32 + lane;      // tile row (token) of this thread
    int ti = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++ti) {
      Tile T;
      decode_tile(A, table, offs, t, T);
      const int ab = ti & 1;
      if (!mbar_wait(&acc_full[ab], (ti >> 1) & 1)) { fail(lane); break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kBN;
      const int hb = ti % kShRing;
      if (!mbar_wait(&sh_full[hb], (ti / kShRing) & 1)) { fail(lane); break; }
      const float* cm = sh + hb * kBN;                 // 2^-e of each weight row of the tile
      float rm = 0.f;                                  // 2^-f of this thread's activation row
      if (row < T.mrows) rm = __ldg(A.rowmul + T.r0 + row);
      if (A.epi == W4_EPI_GELU_GATE) {
        const int Nh = A.N >> 1;
        const int j0 = T.nt * (kBN / 2);
#pragma unroll 1
        for (int c = 0; c < kBN / 2; c += 32) {
          float g[32], u[32];
          tmem_ld32(taddr + c, g);
          tmem_ld32(taddr + kBN / 2 + c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            g[i] = (g[i] * rm) * cm[c + i];
            u[i] = (u[i] * rm) * cm[kBN / 2 + c + i];
          }
          if (row < T.mrows) {
            uint16_t* dst = A.out + (T.r0 + row) * Nh + j0 + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              if (j0 + c + i + 8 <= Nh && (Nh & 7) == 0) {
                uint4 v;
                v.x = pack_bf16x2(gelu_tanh(g[i]) * u[i], gelu_tanh(g[i + 1]) * u[i + 1]);
                v.y = pack_bf16x2(gelu_tanh(g[i + 2]) * u[i + 2], gelu_tanh(g[i + 3]) * u[i + 3]);
                v.z = pack_bf16x2(gelu_tanh(g[i + 4]) * u[i + 4], gelu_tanh(g[i + 5]) * u[i + 5]);
                v.w = pack_bf16x2(gelu_tanh(g[i + 6]) * u[i + 6], gelu_tanh(g[i + 7]) * u[i + 7]);
                *reinterpret_cast<uint4*>(dst + i) = v;
              } else {
                for (int z = 0; z < 8 && j0 + c + i + z < Nh; ++z)
                  dst[i + z] = f32_to_bf16_bits(gelu_tanh(g[i + z]) * u[i + z]);
              }
            }
          }
        }
      } else {
        const int n0 = T.nt * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          float v[32];
          tmem_ld32(taddr + c, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = (v[i] * rm) * cm[c + i];
          if (row < T.mrows) {
            uint16_t* dst = A.out + (T.r0 + row) * A.N + n0 + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              if (n0 + c + i + 8 <= A.N && (A.N & 7) == 0) {
                uint4 w;
                w.x = pack_bf16x2(v[i], v[i + 1]); w.y = pack_bf16x2(v[i + 2], v[i + 3]);
                w.z = pack_bf16x2(v[i + 4], v[i + 5]); w.w = pack_bf16x2(v[i + 6], v[i + 7]);
                *reinterpret_cast<uint4*>(dst + i) = w;
              } else {
                for (int z = 0; z < 8 && n0 + c + i + z < A.N; ++z) dst[i + z] = f32_to_bf16_bits(v[i + z]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh_empty[hb]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  } else if (warp >= 8) {
    // ------------------------------ dequant ------------------------------
    // thread = (weight row r, half hk of the 64-k chunk = one group of 32)
    const int dt = threadIdx.x - 8 * 32;
    const int r = dt & (kBN - 1);
    const int hk = dt >> 7;
    int slot = 0;
    uint32_t fph = 0;       // phase of the full barriers on this lap (the empty ones: fph ^ 1)
    bool lap0 = true;
    int ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
      Tile T;
      decode_tile(A, table, offs, t, T);
      const int sb = ti & 1;
      if (!mbar_wait(&sc_full[sb], (ti >> 1) & 1)) { ok = false; break; }
      const uint32_t* srow = reinterpret_cast<const uint32_t*>(smem + Smem::sc + sb * kScaleBytes) +
                             r * ((A.kg >> 1) | 1);
      // row exponent e: the row's largest finite |scale| lands in [2^11, 2^12), so |s * 2^e * q|
      // stays below 2^15 and every scale within 2^28 of the largest keeps s * 2^e * q exact
      uint32_t m = 0;
      for (int j = 0; j < (A.kg >> 1); ++j) {
        const uint32_t v = srow[j];
        const uint32_t lo = v & 0x7FFFu, hi = (v >> 16) & 0x7FFFu;
        if (lo < 0x7F80u) m = max(m, lo);
        if (hi < 0x7F80u) m = max(m, hi);
      }
      const int e = shift_for(m, 11);
      const float smul = pow2f(e);
      if (hk == 0) {
        const int hb = ti % kShRing;
        if (ti >= kShRing && !mbar_wait(&sh_empty[hb], ((ti / kShRing) - 1) & 1)) { ok = false; break; }
        sh[hb * kBN + r] = pow2f(-e);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh_full[hb]);
      }
      for (int kc = 0; kc < nk; ++kc) {
        if (!mbar_wait(&raw_full[slot], fph)) { ok = false; break; }
        const uint4 w = *reinterpret_cast<const uint4*>(smem + Smem::raw + slot * kRawBytes + r * 32 + hk * 16);
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[slot]);
        const float sf = bf16_lo_to_f32(srow[kc] >> (16 * hk)) * smul;      // group g = 2 kc + hk
        const __half2 sh2 = __float2half2_rn(sf);
        const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&sh2);
        uint32_t pk[16];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pk[4 * i + 0] = f16x2_mul(nibbles_to_f16x2(ww[i]), s2);        // elements 8i+0,1
          pk[4 * i + 1] = f16x2_mul(nibbles_to_f16x2(ww[i] >> 4), s2);   // 8i+2,3
          pk[4 * i + 2] = f16x2_mul(nibbles_to_f16x2(ww[i] >> 8), s2);   // 8i+4,5
          pk[4 * i + 3] = f16x2_mul(nibbles_to_f16x2(ww[i] >> 12), s2);  // 8i+6,7
        }
        if (!lap0 && !mbar_wait(&ab_empty[slot], fph ^ 1u)) { ok = false; break; }
        const uint32_t bbase = smem_u32(smem + Smem::b + slot * kBBytes) + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = hk * 4 + i;                      // 16-byte chunk = elements 8c..8c+7
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(bbase + ((c ^ (r & 7)) << 4)), "r"(pk[4 * i]), "r"(pk[4 * i + 1]),
                         "r"(pk[4 * i + 2]), "r"(pk[4 * i + 3]) : "memory");
        }
        fence_proxy_async();                              // generic writes -> async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&b_full[slot]);
        if (++slot == kStages) { slot = 0; fph ^= 1u; lap0 = false; }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sc_empty[sb]);
    }
    if (!ok) fail(lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace tc
}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static size_t tc_smem_bytes(int E) { return w4::tc::Smem::table + static_cast<size_t>(E + 1) * 8 + 1024; }

bool w4_tc_supported(int N, int K, int epi) {
  const int kg = K / 32;
  if (kg > w4::tc::kMaxKg || kg % 2) return false;            // scale block fits; 64-k chunks
  if (epi == W4_EPI_GELU_GATE) return (N / 2) % (w4::tc::kBN / 2) == 0;
  return N % w4::tc::kBN == 0;
}

// fp16 activation rows in pair order [rows, K], then the row multipliers [rows]
size_t w4_tc_workspace_bytes(int64_t rows, int K) {
  if (rows <= 0) return 0;
  return (static_cast<size_t>(rows) * K * 2 + 255) / 256 * 256 + static_cast<size_t>(rows) * 4;
}

w4_status w4_launch_tc_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                            const uint32_t* codes, const uint16_t* scales, const int32_t* offsets,
                            int E, int64_t rows, int N, int K, int epi, uint16_t* out, void* ws,
                            size_t ws_bytes, int32_t* dev_status, cudaStream_t stream, int sm_count) {
  if (!w4_tc_supported(N, K, epi)) return W4_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(scales) & 15) != 0) return W4_ERR_UNSUPPORTED;
  if (rows == 0) return W4_OK;
  w4::tc::TcArgs A{};
  const int kd = k_div > 0 ? k_div : 1;
  const int64_t a_rows = a_row_of_pair ? rows / kd : rows;   // rows of `a` a pair may name
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32; A.rows = rows;
  A.epi = epi; A.out = out;
  A.n_tiles = (epi == W4_EPI_GELU_GATE) ? (N / 2) / (w4::tc::kBN / 2) : N / w4::tc::kBN;
  A.dev_status = dev_status;
  if (a_rows <= 0) return W4_ERR_INVALID_ARG;
  if (!ws || ws_bytes < w4_tc_workspace_bytes(rows, K) || (reinterpret_cast<uintptr_t>(ws) & 15))
    return W4_ERR_WORKSPACE;
  uint16_t* a16 = static_cast<uint16_t*>(ws);
  float* rowmul = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                           (static_cast<size_t>(rows) * K * 2 + 255) / 256 * 256);
  A.rowmul = rowmul;
  {
    const int64_t blocks = (rows + 7) / 8;
    const int grid = static_cast<int>(blocks < 16LL * sm_count ? blocks : 16LL * sm_count);
    w4::tc::a_to_f16_kernel<<<grid, 256, 0, stream>>>(a, a_row_of_pair, kd, a_rows, rows, K, a16,
                                                      rowmul, dev_status);
  }
  // raw codes: [E*N, K/8] words, box = 8 words (one 64-k chunk) x 64 rows, no swizzle
  auto fn = tc_encode_fn();
  if (!fn) return W4_ERR_CUDA;
  CUtensorMap tmap;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 8), static_cast<cuuint64_t>(E) * N};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 8) * 4};
  cuuint32_t box[2] = {8, static_cast<cuuint32_t>(w4::tc::kBN / 2)};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return W4_ERR_CUDA;
  // converted activations [rows, K] fp16: box = 64 k x 128 rows, 128-byte swizzle
  CUtensorMap amap;
  cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t astr[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t abox[2] = {static_cast<cuuint32_t>(w4::tc::kBK), static_cast<cuuint32_t>(w4::tc::kBM)};
  if (fn(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a16, adims, astr, abox, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return W4_ERR_CUDA;
  const size_t smem = tc_smem_bytes(E);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::tc::tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes(1024))) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  w4::tc::tc_gemm_kernel<<<sm_count, w4::tc::kThreads, smem, stream>>>(tmap, amap, A);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
