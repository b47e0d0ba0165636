// Weight-streaming W4A16 GEMM for few tokens per weight matrix (decode, dense GEMV-like linears,
// lightly loaded experts).
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "What changed in vLLM's TPU backend": the grouped matmul takes a scale per 32-wide group and
// dequantises each weight tile in on-chip memory before the multiply; activations stay bf16.
// Decode re-reads every active weight per step, so this path is bound by HBM bandwidth
// ("Compression Without Regret: Quantization, QAT, and Shipping Smaller Models", section
// "1. Why quantization pays off").
//
// Design (sm_100a):
//   * Work unit = (expert e, token block of <= 32 routed rows, tile of 128 weight rows, K split).
//     A persistent grid (one CTA per SM) walks the units; the unit table is a prefix sum over
//     experts built on the device from expert_offsets, so no host synchronisation is needed.
//   * One producer warp feeds a 4-stage shared-memory ring: per stage 8 groups (256 k) of the
//     128-row code tile by a 2-D TMA copy with the 128-byte swizzle (two 64-row boxes), the
//     matching bf16 scales by 4-byte cp.async, and the <= 32 activation rows (gathered by
//     a_row_of_pair) by 1-D bulk copies, all completing on one mbarrier.
//   * Eight consumer warps each own 16 weight rows.  A thread's 32-bit code word is turned into
//     four bf16 pairs (one lop3 + one packed fma per pair), which are exactly the A fragments of
//     two m16n8k16 MMAs, with the tokens as the n = 8 side.  The MMA's k order is permuted so
//     that word t of a group feeds quad position t; the activation pairs are permuted to match
//     with prmt.  Each group's two MMAs start from zero and the group's bf16 scale is folded in
//     with one fp32 FMA per accumulator: acc += s_g * (sum over the group of q * x).  Products
//     q * x are exact in fp32.
//   * Epilogue through shared memory: bf16 rows, the GELU gate (gate rows in warps 0-3, up rows
//     in warps 4-7 of the same tile), or float32 split-K partials reduced in a fixed order by
//     the last CTA of the tile (deterministic).
#include <cudaTypedefs.h>

#include "common.cuh"

namespace w4 {

constexpr int kStages = 4;
constexpr int kGS = 8;                        // groups per stage
constexpr int kCWarps = 8;                    // consumer warps
constexpr int kBN = 16 * kCWarps;             // weight rows per tile
constexpr int kHalf = kBN / 2;                // rows per TMA box
constexpr int kMT = 32;                       // routed rows (tokens) per unit
constexpr int kXPitch = kGS * 64 + 64;        // bytes per token row in an activation stage
constexpr int kCodeBytes = kBN * kGS * 16;    // 16 KB
constexpr int kXBytes = kMT * kXPitch;        // 18 KB
constexpr int kScaleBytes = kBN * kGS * 2;    // 2 KB
constexpr int kEpPitch = kBN + 4;             // floats per token row in the epilogue buffer
constexpr int kThreads = (kCWarps + 1) * 32;

struct StreamArgs {
  const uint16_t* a;
  const int32_t* a_row_of_pair;
  int k_div;
  const uint16_t* scales;   // [E*N, kg]
  const int32_t* offsets;   // [E+1] or null (one expert with `rows` rows)
  int E, N, K, kg;
  int64_t rows;
  int64_t a_rows;           // rows of `a` (gathered row indices are checked against it)
  int epi;
  uint16_t* out;
  float* partial;           // [splits, rows, N] (splits > 1)
  int32_t* counters;        // [tiles] (splits > 1)
  int splits, stages_per_split, n_tiles;
  int scale_mode;           // 1: producer cp.async (kg even); 0: consumers load from global
  int32_t* dev_status;
};

struct SmemLayout {
  static constexpr int codes = 0;
  static constexpr int x = codes + kStages * kCodeBytes;
  static constexpr int sc = x + kStages * kXBytes;
  static constexpr int ep = sc + kStages * kScaleBytes;
  static constexpr int bars = ep + kMT * kEpPitch * 4;
  static constexpr int flags = bars + 2 * kStages * 8;
  static constexpr int table = flags + 16;        // int table[E + 1], then int offs[E + 1]
  static constexpr int bytes_without_table = table;
};

struct Unit {
  int e, tb, nt, sp;
  int64_t r0;
  int mt;
  int g0, g1;
};

// Unit u -> (expert, token block, tile, split); `table` and `offs` live in shared memory.
__device__ __forceinline__ void decode_unit(const StreamArgs& A, const int* table, const int* offs,
                                            int64_t u, Unit& U) {
  int lo = 0, hi = A.E - 1;                       // largest e with table[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (table[mid] <= u) lo = mid; else hi = mid - 1;
  }
  U.e = lo;
  const int64_t off0 = offs[U.e], off1 = offs[U.e + 1];
  const int ntb = max(1, static_cast<int>((off1 - off0 + kMT - 1) / kMT));
  const int64_t local = u - table[U.e];
  U.tb = static_cast<int>(local % ntb);
  const int64_t rest = local / ntb;
  U.sp = static_cast<int>(rest % A.splits);
  U.nt = static_cast<int>(rest / A.splits);
  U.r0 = off0 + static_cast<int64_t>(U.tb) * kMT;
  U.mt = static_cast<int>(off1 - U.r0 < kMT ? off1 - U.r0 : kMT);
  U.g0 = U.sp * A.stages_per_split * kGS;
  U.g1 = min(A.kg, U.g0 + A.stages_per_split * kGS);
}

// global weight row (e*N + n) of tile row r in [0, kBN)
__device__ __forceinline__ int64_t tile_row(const StreamArgs& A, const Unit& U, int r) {
  int n;
  if (A.epi == W4_EPI_GELU_GATE) {
    const int j = U.nt * kHalf + (r & (kHalf - 1));
    n = (r < kHalf) ? j : (A.N >> 1) + j;
  } else {
    n = U.nt * kBN + r;
  }
  return static_cast<int64_t>(U.e) * A.N + n;
}

__device__ __forceinline__ bool tile_row_valid(const StreamArgs& A, const Unit& U, int r) {
  if (A.epi == W4_EPI_GELU_GATE) return U.nt * kHalf + (r & (kHalf - 1)) < (A.N >> 1);
  return U.nt * kBN + r < A.N;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32) : "memory");
}

// Source row in `a` of routed row r (checked; out-of-range indices read row 0 and are reported).
__device__ __forceinline__ int64_t gather_row(const StreamArgs& A, int64_t r) {
  int64_t src = A.a_row_of_pair ? static_cast<int64_t>(__ldg(A.a_row_of_pair + r) / A.k_div) : r;
  if (src < 0 || src >= A.a_rows) {
    set_status(A.dev_status, W4_ERR_INVALID_ARG);
    src = 0;
  }
  return src;
}

__global__ void __launch_bounds__(kThreads, 1)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes, StreamArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars);
  uint64_t* empty = full + kStages;
  volatile int* flags = reinterpret_cast<volatile int*>(smem + SmemLayout::flags);
  int* table = reinterpret_cast<int*>(smem + SmemLayout::table);
  int* offs = table + (A.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Activation stages start zeroed: groups past a K tail read finite (stale or zero) values
  // that meet a zero scale.
  for (int i = threadIdx.x; i < kStages * kXBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + SmemLayout::x)[i] = make_uint4(0, 0, 0, 0);

  // unit table: table[e] = first unit of expert e, table[E] = total; offsets copied to offs[].
  // Offsets that are not non-decreasing from 0 to rows make the launch a no-op (W4_ERR_INVALID_ARG).
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
        const int64_t ntb = o1 > o0 ? (o1 - o0 + kMT - 1) / kMT : 0;
        cnt = static_cast<int>(ntb * A.n_tiles * A.splits);
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
      mbar_init(&full[s], 1 + (A.scale_mode ? 32 : 0));
      mbar_init(&empty[s], kCWarps);
    }
    flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t total_units = table[A.E];

  if (warp == kCWarps) {
    // ------------------------------- producer -------------------------------
    if (lane == 0) prefetch_tmap(&tmap_codes);
    uint32_t it = 0;
    int64_t u = blockIdx.x;
    Unit U;
    int64_t src_row = 0;
    if (u < total_units) {
      decode_unit(A, table, offs, u, U);
      if (lane < U.mt) src_row = gather_row(A, U.r0 + lane);
    }
    while (u < total_units) {
      // prefetch the next unit's gather rows while this unit's stages are issued
      const int64_t un = u + gridDim.x;
      Unit Un;
      int64_t src_next = 0;
      if (un < total_units) {
        decode_unit(A, table, offs, un, Un);
        if (lane < Un.mt) src_next = gather_row(A, Un.r0 + lane);
      }
      const int64_t row_a = tile_row(A, U, 0);
      const int64_t row_b = tile_row(A, U, kHalf);
      for (int g = U.g0; g < U.g1; g += kGS, ++it) {
        const int slot = it % kStages;
        const uint32_t round = it / kStages;
        const int gc = min(kGS, U.g1 - g);
        if (round > 0) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&empty[slot], (round - 1) & 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok || flags[0]) {
            if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
            return;
          }
        }
        uint8_t* cdst = smem + SmemLayout::codes + slot * kCodeBytes;
        uint8_t* xdst = smem + SmemLayout::x + slot * kXBytes;
        const uint32_t xbytes = static_cast<uint32_t>(gc) * 64u;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[slot], kCodeBytes + xbytes * U.mt);
          tma_load_2d(cdst, &tmap_codes, g * 4, static_cast<int32_t>(row_a), &full[slot]);
          tma_load_2d(cdst + kHalf * 128, &tmap_codes, g * 4, static_cast<int32_t>(row_b), &full[slot]);
        }
        __syncwarp();
        if (lane < U.mt)
          bulk_g2s(xdst + lane * kXPitch, A.a + src_row * A.K + static_cast<int64_t>(g) * 32, xbytes,
                   &full[slot]);
        if (A.scale_mode) {
          const uint32_t sdst = smem_u32(smem + SmemLayout::sc + slot * kScaleBytes);
#pragma unroll 1
          for (int r = lane; r < kBN; r += 32) {
            const int64_t grow = tile_row_valid(A, U, r) ? tile_row(A, U, r) : row_a;
            const uint16_t* src = A.scales + grow * A.kg + g;
            for (int p = 0; p < gc; p += 2) cp_async4(sdst + r * 16 + p * 2, src + p);
          }
          cp_async_arrive_noinc(&full[slot]);
        }
      }
      u = un;
      U = Un;
      src_row = src_next;
    }
    return;
  }

  // ------------------------------- consumers -------------------------------
  const int gid = lane >> 2, tq = lane & 3;
  const int rlo = warp * 16 + gid, rhi = rlo + 8;
  float* ep = reinterpret_cast<float*>(smem + SmemLayout::ep);
  uint32_t it = 0;
  bool aborted = false;   // after a timed-out wait: skip work, keep every barrier
  for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
    Unit U;
    decode_unit(A, table, offs, u, U);
    const int nblk = (U.mt + 7) >> 3;
    float acc[4][4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;
    const int64_t grow_lo = tile_row_valid(A, U, rlo) ? tile_row(A, U, rlo) : tile_row(A, U, 0);
    const int64_t grow_hi = tile_row_valid(A, U, rhi) ? tile_row(A, U, rhi) : tile_row(A, U, 0);

    for (int g = U.g0; g < U.g1; g += kGS, ++it) {
      const int slot = it % kStages;
      const uint32_t round = it / kStages;
      const int gc = min(kGS, U.g1 - g);
      if (!aborted && (!mbar_wait(&full[slot], round & 1) || flags[0])) {
        if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
        aborted = true;
      }
      if (aborted) continue;
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(smem + SmemLayout::codes + slot * kCodeBytes);
      const uint8_t* xs = smem + SmemLayout::x + slot * kXBytes;
      uint32_t slo[4], shi[4];
      if (A.scale_mode) {
        const uint4* sc = reinterpret_cast<const uint4*>(smem + SmemLayout::sc + slot * kScaleBytes);
        const uint4 vlo = sc[rlo], vhi = sc[rhi];
        slo[0] = vlo.x; slo[1] = vlo.y; slo[2] = vlo.z; slo[3] = vlo.w;
        shi[0] = vhi.x; shi[1] = vhi.y; shi[2] = vhi.z; shi[3] = vhi.w;
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int ga = g + 2 * p, gb = g + 2 * p + 1;
          const uint32_t l0 = ga < U.g1 ? ldg_u16(A.scales + grow_lo * A.kg + ga) : 0;
          const uint32_t l1 = gb < U.g1 ? ldg_u16(A.scales + grow_lo * A.kg + gb) : 0;
          const uint32_t h0 = ga < U.g1 ? ldg_u16(A.scales + grow_hi * A.kg + ga) : 0;
          const uint32_t h1 = gb < U.g1 ? ldg_u16(A.scales + grow_hi * A.kg + gb) : 0;
          slo[p] = l0 | (l1 << 16);
          shi[p] = h0 | (h1 << 16);
        }
      }
      // Dequantise the stage's 8 groups for rows rlo / rhi into MMA A fragments.  The word of
      // row r, group gi, quad position tq sits at chunk (gi ^ r%8) of the row (128-byte swizzle).
      uint32_t fa[kGS][8];
      float fsl[kGS], fsh[kGS];
#pragma unroll
      for (int gi = 0; gi < kGS; ++gi) {
        const uint32_t wlo = cw[rlo * 32 + ((gi ^ (rlo & 7)) << 2) + tq];
        const uint32_t whi = cw[rhi * 32 + ((gi ^ (rhi & 7)) << 2) + tq];
        fa[gi][0] = nibbles_to_bf16x2(wlo);        // k-step 0: nibbles (0,4) | (1,5)
        fa[gi][1] = nibbles_to_bf16x2(whi);
        fa[gi][2] = nibbles_to_bf16x2(wlo >> 4);
        fa[gi][3] = nibbles_to_bf16x2(whi >> 4);
        fa[gi][4] = nibbles_to_bf16x2(wlo >> 8);   // k-step 1: nibbles (2,6) | (3,7)
        fa[gi][5] = nibbles_to_bf16x2(whi >> 8);
        fa[gi][6] = nibbles_to_bf16x2(wlo >> 12);
        fa[gi][7] = nibbles_to_bf16x2(whi >> 12);
        const uint32_t sl = (gi & 1) ? (slo[gi >> 1] & 0xFFFF0000u) : (slo[gi >> 1] << 16);
        const uint32_t sh = (gi & 1) ? (shi[gi >> 1] & 0xFFFF0000u) : (shi[gi >> 1] << 16);
        fsl[gi] = gi < gc ? __uint_as_float(sl) : 0.f;   // groups past the K range add nothing
        fsh[gi] = gi < gc ? __uint_as_float(sh) : 0.f;
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (b < nblk) {
          const uint8_t* xrow = xs + (b * 8 + gid) * kXPitch + tq * 16;
#pragma unroll
          for (int gi = 0; gi < kGS; ++gi) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xrow + gi * 64);
            const uint32_t b00 = prmt(xv.x, xv.z, 0x5410), b01 = prmt(xv.x, xv.z, 0x7632);
            const uint32_t b10 = prmt(xv.y, xv.w, 0x5410), b11 = prmt(xv.y, xv.w, 0x7632);
            const uint32_t a0[4] = {fa[gi][0], fa[gi][1], fa[gi][2], fa[gi][3]};
            const uint32_t a1[4] = {fa[gi][4], fa[gi][5], fa[gi][6], fa[gi][7]};
            float d[4];
            const float z[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16_16816(d, a0, b00, b01, z);
            mma_bf16_16816(d, a1, b10, b11, d);
            acc[b][0] = fmaf(fsl[gi], d[0], acc[b][0]);
            acc[b][1] = fmaf(fsl[gi], d[1], acc[b][1]);
            acc[b][2] = fmaf(fsh[gi], d[2], acc[b][2]);
            acc[b][3] = fmaf(fsh[gi], d[3], acc[b][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // --------------------------- epilogue ---------------------------
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nblk) {
        const int t0 = b * 8 + 2 * tq;
        ep[t0 * kEpPitch + rlo] = acc[b][0];
        ep[(t0 + 1) * kEpPitch + rlo] = acc[b][1];
        ep[t0 * kEpPitch + rhi] = acc[b][2];
        ep[(t0 + 1) * kEpPitch + rhi] = acc[b][3];
      }
    }
    consumer_sync();
    const int ctid = threadIdx.x;  // 0..255
    if (flags[0]) {
      // aborted CTA: write nothing, keep the barrier count of the normal path
      if (A.epi != W4_EPI_GELU_GATE && A.splits > 1) { consumer_sync(); consumer_sync(); }
    } else if (A.epi == W4_EPI_GELU_GATE) {
      const int Nh = A.N >> 1;
      const int j0 = U.nt * kHalf;
      for (int idx = ctid; idx < U.mt * (kHalf / 8); idx += kCWarps * 32) {
        const int t = idx / (kHalf / 8), c = idx % (kHalf / 8);
        const float* gp = ep + t * kEpPitch + c * 8;
        const float* up = gp + kHalf;
        float h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = gelu_tanh(gp[i]) * up[i];
        uint16_t* dst = A.out + (U.r0 + t) * Nh + j0 + c * 8;
        if (j0 + c * 8 + 8 <= Nh && (Nh & 7) == 0) {
          uint4 v;
          v.x = pack_bf16x2(h[0], h[1]); v.y = pack_bf16x2(h[2], h[3]);
          v.z = pack_bf16x2(h[4], h[5]); v.w = pack_bf16x2(h[6], h[7]);
          *reinterpret_cast<uint4*>(dst) = v;
        } else {
          for (int i = 0; i < 8 && j0 + c * 8 + i < Nh; ++i) dst[i] = f32_to_bf16_bits(h[i]);
        }
      }
    } else if (A.splits == 1) {
      const int n0 = U.nt * kBN;
      for (int idx = ctid; idx < U.mt * (kBN / 8); idx += kCWarps * 32) {
        const int t = idx / (kBN / 8), c = idx % (kBN / 8);
        const float* src = ep + t * kEpPitch + c * 8;
        uint16_t* dst = A.out + (U.r0 + t) * A.N + n0 + c * 8;
        if (n0 + c * 8 + 8 <= A.N && (A.N & 7) == 0) {
          uint4 v;
          v.x = pack_bf16x2(src[0], src[1]); v.y = pack_bf16x2(src[2], src[3]);
          v.z = pack_bf16x2(src[4], src[5]); v.w = pack_bf16x2(src[6], src[7]);
          *reinterpret_cast<uint4*>(dst) = v;
        } else {
          for (int i = 0; i < 8 && n0 + c * 8 + i < A.N; ++i) dst[i] = f32_to_bf16_bits(src[i]);
        }
      }
    } else {
      // split-K: float32 partial, then the last CTA of the tile reduces in split order
      const int n0 = U.nt * kBN;
      for (int idx = ctid; idx < U.mt * kBN; idx += kCWarps * 32) {
        const int t = idx / kBN, c = idx % kBN;
        if (n0 + c < A.N)
          A.partial[(static_cast<int64_t>(U.sp) * A.rows + U.r0 + t) * A.N + n0 + c] = ep[t * kEpPitch + c];
      }
      __threadfence();
      consumer_sync();
      if (ctid == 0) {
        const int tile = U.tb * A.n_tiles + U.nt;
        const int prev = atomicAdd(&A.counters[tile], 1);
        const int last = (prev == A.splits - 1);
        if (last) A.counters[tile] = 0;
        flags[1] = last;
      }
      consumer_sync();
      if (flags[1]) {
        __threadfence();
        for (int idx = ctid; idx < U.mt * kBN; idx += kCWarps * 32) {
          const int t = idx / kBN, c = idx % kBN;
          if (n0 + c < A.N) {
            float s = 0.f;
            for (int sp = 0; sp < A.splits; ++sp)
              s += __ldcg(&A.partial[(static_cast<int64_t>(sp) * A.rows + U.r0 + t) * A.N + n0 + c]);
            A.out[(U.r0 + t) * A.N + n0 + c] = f32_to_bf16_bits(s);
          }
        }
      }
    }
    consumer_sync();
  }
}

}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

// Codes [rows_total, K/8] uint32 as a 2-D tensor: box = 32 words x 64 rows, 128-byte swizzle.
static bool encode_codes_map(CUtensorMap* m, const uint32_t* codes, int64_t rows_total, int K) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 8), static_cast<cuuint64_t>(rows_total)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 8) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(w4::kHalf)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static size_t stream_smem_bytes(int E) {
  return w4::SmemLayout::bytes_without_table + static_cast<size_t>(E + 1) * 8 + 1024;
}

struct StreamPlan {
  int splits, stages_per_split, n_tiles;
};

static StreamPlan plan_stream(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  StreamPlan p;
  const int kg = K / 32;
  const int kstages = (kg + w4::kGS - 1) / w4::kGS;
  p.n_tiles = (epi == W4_EPI_GELU_GATE) ? ((N / 2) + w4::kHalf - 1) / w4::kHalf
                                        : (N + w4::kBN - 1) / w4::kBN;
  p.splits = 1;
  if (dense) {
    // split K while the units do not fill the SMs four times over and the float32 partials stay
    // below ~1/8 of the weight bytes
    const int64_t ntb = (rows + w4::kMT - 1) / w4::kMT;
    const double wbytes = static_cast<double>(N) * K * 0.5625;
    while (p.splits * 2 <= kstages && ntb * p.n_tiles * p.splits < 4LL * sm_count &&
           static_cast<double>(p.splits * 2) * rows * N * 8.0 <= wbytes / 8.0)
      p.splits *= 2;
  }
  p.stages_per_split = (kstages + p.splits - 1) / p.splits;
  p.splits = (kstages + p.stages_per_split - 1) / p.stages_per_split;
  return p;
}

size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  if (p.splits == 1) return 0;
  const int64_t ntb = (rows + w4::kMT - 1) / w4::kMT;
  size_t b = static_cast<size_t>(p.splits) * rows * N * sizeof(float);
  b = (b + 255) & ~size_t(255);
  return b + static_cast<size_t>(ntb * p.n_tiles) * sizeof(int32_t);
}

w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count) {
  const bool dense = (offsets == nullptr);
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  w4::StreamArgs A{};
  A.a = a; A.a_row_of_pair = a_row_of_pair; A.k_div = k_div > 0 ? k_div : 1;
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32; A.rows = rows; A.epi = epi; A.out = out;
  A.a_rows = a_row_of_pair ? rows / A.k_div : rows;
  A.splits = p.splits; A.stages_per_split = p.stages_per_split; A.n_tiles = p.n_tiles;
  A.scale_mode = (A.kg % 2 == 0) ? 1 : 0;
  A.dev_status = dev_status;
  if (p.splits > 1) {
    const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count);
    if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
    size_t pb = static_cast<size_t>(p.splits) * rows * N * sizeof(float);
    pb = (pb + 255) & ~size_t(255);
    A.partial = static_cast<float*>(ws);
    A.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + pb);
  }
  if (rows == 0) return W4_OK;
  CUtensorMap tmap;
  if (!encode_codes_map(&tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  const size_t smem = stream_smem_bytes(E);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(stream_smem_bytes(1024))) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  w4::stream_gemm_kernel<<<sm_count, w4::kThreads, smem, stream>>>(tmap, A);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
