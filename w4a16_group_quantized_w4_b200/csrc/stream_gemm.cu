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
//   * Work unit = (expert e, block of <= MT routed rows (MT = 8 or 16), tile of 128 weight rows,
//     K split).  A persistent grid (two CTAs per SM) walks the units; the unit table is a prefix
//     sum over the experts built on the device from expert_offsets (no host synchronisation).
//   * Each CTA = 8 compute warps + 1 producer warp.  The producer keeps a shared-memory ring as
//     deep as the per-CTA shared-memory budget allows (4-6 stages) full: one stage = 8 groups
//     (256 k) of the 128-row code tile (two 64-row 2-D TMA boxes, 128-byte swizzle), the matching
//     bf16 scales (two 2-D TMA boxes when a scale row is a whole number of 16-byte chunks, else the
//     tile's contiguous 64-row scale blocks by 1-D bulk copy), and the activation rows gathered by
//     a_row_of_pair (1-D bulk copies).  Everything completes on the stage's mbarrier.
//   * A compute warp owns 16 weight rows.  A thread's 32-bit code word becomes four bf16 pairs
//     128 + u (one lop3 per pair, exact), which are exactly the A fragments of two m16n8k16 MMAs
//     with the tokens as the n = 8 side; two more MMAs with the constant A = -136 remove the bias
//     (q = u - 8).  The packed nibble order puts two consecutive k in each extracted pair, so the
//     activation B fragments are plain 16-byte shared loads.  Each group's MMAs start from zero
//     and the group's scale is folded in with one fp32 FMA per accumulator:
//     acc += s_g * (sum over the group of q * x).  Products q * x are exact in fp32.
//   * Epilogue from registers, without a CTA barrier: with the GELU gate each warp's two A-fragment
//     row sets are 8 gate rows and the 8 up rows of the same outputs, so h = gelu(g) * u is formed
//     in the thread that holds both.  Dense split-K writes float32 partials that the last CTA of
//     the tile reduces in a fixed order (deterministic).
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"

namespace w4 {

#ifndef W4_STREAM_GROUPS_PER_PASS
#define W4_STREAM_GROUPS_PER_PASS 4           // groups dequantised into registers at a time
#endif
#ifndef W4_STREAM_BIASED
#define W4_STREAM_BIASED 0                    // 1: codes as 128 + u plus a -136 MMA; 0: u - 8 by fma
#endif

constexpr int kMaxStages = 6;
constexpr int kGS = 8;                        // groups per stage
constexpr int kGP = W4_STREAM_GROUPS_PER_PASS;
constexpr int kWarps = 8;                     // compute warps
constexpr int kThreads = (kWarps + 1) * 32;   // + one producer warp
constexpr int kBN = 16 * kWarps;              // weight rows per tile
constexpr int kHalf = kBN / 2;                // rows per TMA box
constexpr int kXPitch = kGS * 64 + 64;        // bytes per token row in an activation stage
constexpr int kCodeBytes = kBN * kGS * 16;    // 16 KB
constexpr int kBlockMaxKg = 24;               // scale-block mode: two 64-row blocks of <= 24 groups
constexpr int kEpPitch = kBN + 4;             // floats per token row in the epilogue buffer
constexpr int kCtasPerSm = 2;
// shared memory one CTA may use when two share an SM (228 KB per SM, 1 KB reserved per CTA)
constexpr int kSmemPerCta = (233472 - kCtasPerSm * 1024) / kCtasPerSm;

enum ScaleMode { kScaleLdg = 0, kScaleBlock = 1, kScaleTma = 2 };

// Shared-memory layout, fixed per launch (offsets from the 1024-byte aligned base).
struct Layout {
  int stages;
  int x_off, x_bytes;        // activation ring: stages x (MT rows x kXPitch)
  int sc_off, sc_bytes;      // scale ring: stages x sc_bytes
  int ep_off;                // split-K epilogue buffer (MT x kEpPitch floats), or -1
  int bar_off;               // 2 * stages mbarriers
  int flag_off;              // 16 bytes
  int table_off;             // int table[E + 1], int offs[E + 1]
  int total;
};

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
  int scale_mode;
  Layout L;
  int32_t* dev_status;
};

struct Unit {
  int e, tb, nt, sp;
  int64_t r0;
  int mt;
  int g0, g1;
};

// Unit u -> (expert, token block, tile, split); `table` and `offs` live in shared memory.
template <int MT>
__device__ __forceinline__ void decode_unit(const StreamArgs& A, const int* table, const int* offs,
                                            int64_t u, Unit& U) {
  int lo = 0, hi = A.E - 1;                       // largest e with table[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (table[mid] <= u) lo = mid; else hi = mid - 1;
  }
  U.e = lo;
  const int off0 = offs[U.e], off1 = offs[U.e + 1];
  const int ntb = max(1, (off1 - off0 + MT - 1) / MT);
  const int local = static_cast<int>(u) - table[U.e];      // 32-bit: unit counts fit in int
  int rest;
  if (ntb == 1) { U.tb = 0; rest = local; }
  else { rest = local / ntb; U.tb = local - rest * ntb; }
  if (A.splits == 1) { U.sp = 0; U.nt = rest; }
  else { U.nt = rest / A.splits; U.sp = rest - U.nt * A.splits; }
  U.r0 = off0 + U.tb * MT;
  U.mt = min(MT, off1 - static_cast<int>(U.r0));
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

// Source row in `a` of routed row r (checked; out-of-range indices read row 0 and are reported).
__device__ __forceinline__ int64_t gather_row(const StreamArgs& A, int64_t r) {
  int64_t src = A.a_row_of_pair ? static_cast<int64_t>(__ldg(A.a_row_of_pair + r) / A.k_div) : r;
  if (src < 0 || src >= A.a_rows) {
    set_status(A.dev_status, W4_ERR_INVALID_ARG);
    src = 0;
  }
  return src;
}

// Barrier over the compute warps only (the producer warp never joins it).
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
}

template <int MT, bool GELU>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, StreamArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (128-byte swizzle atoms), derived by pointer arithmetic so that every
  // pointer below stays in the shared address space (plain shared loads, not generic ones)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Layout& L = A.L;
  const int S = L.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + S;
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flag_off);
  int* table = reinterpret_cast<int*>(smem + L.table_off);
  int* offs = table + (A.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Activation stages start zeroed: groups past a K tail read finite (stale or zero) values
  // that meet a zero scale.
  for (int i = threadIdx.x; i < S * L.x_bytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + L.x_off)[i] = make_uint4(0, 0, 0, 0);

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
        const int64_t ntb = o1 > o0 ? (o1 - o0 + MT - 1) / MT : 0;
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
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t total_units = table[A.E];

  if (warp == kWarps) {
    // ------------------------------- producer -------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_codes);
      if (A.scale_mode == kScaleTma) prefetch_tmap(&tmap_scales);
    }
    int slot = 0;
    uint32_t phase = 0;        // phase of the empty barrier to wait for on the next lap
    bool first_lap = true;
    for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
      Unit U;
      decode_unit<MT>(A, table, offs, u, U);
      const int64_t src_row = lane < U.mt ? gather_row(A, U.r0 + lane) : 0;
      const int64_t row_a = tile_row(A, U, 0);
      const int64_t row_b = tile_row(A, U, kHalf);
      for (int g = U.g0; g < U.g1; g += kGS) {
        if (!first_lap) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&empty[slot], phase);
          if (!__shfl_sync(0xffffffffu, ok, 0) || flags[0]) {
            if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
            return;
          }
        }
        const int gc = min(kGS, U.g1 - g);
        uint8_t* cdst = smem + slot * kCodeBytes;
        uint8_t* xdst = smem + L.x_off + slot * L.x_bytes;
        uint8_t* sdst = smem + L.sc_off + slot * L.sc_bytes;
        const uint32_t xbytes = static_cast<uint32_t>(gc) * 64u;
        if (lane == 0) {
          uint32_t sbytes = 0;
          if (A.scale_mode == kScaleTma) sbytes = 2 * kHalf * kGS * 2;
          else if (A.scale_mode == kScaleBlock) sbytes = 2 * kHalf * A.kg * 2;
          mbar_arrive_expect_tx(&full[slot], kCodeBytes + sbytes + xbytes * U.mt);
          tma_load_2d(cdst, &tmap_codes, g * 4, static_cast<int32_t>(row_a), &full[slot]);
          tma_load_2d(cdst + kHalf * 128, &tmap_codes, g * 4, static_cast<int32_t>(row_b), &full[slot]);
          if (A.scale_mode == kScaleTma) {
            tma_load_2d(sdst, &tmap_scales, g, static_cast<int32_t>(row_a), &full[slot]);
            tma_load_2d(sdst + kHalf * kGS * 2, &tmap_scales, g, static_cast<int32_t>(row_b), &full[slot]);
          } else if (A.scale_mode == kScaleBlock) {
            const uint32_t blk = kHalf * A.kg * 2;
            bulk_g2s(sdst, A.scales + row_a * A.kg, blk, &full[slot]);
            bulk_g2s(sdst + blk, A.scales + row_b * A.kg, blk, &full[slot]);
          }
        }
        __syncwarp();
        if (lane < U.mt)
          bulk_g2s(xdst + lane * kXPitch, A.a + src_row * A.K + static_cast<int64_t>(g) * 32, xbytes,
                   &full[slot]);
        if (++slot == S) { slot = 0; if (!first_lap) phase ^= 1u; first_lap = false; }
      }
    }
    return;
  }

  // ------------------------------- compute warps -------------------------------
  // Rows of this thread's two A-fragment rows.  GELU gate: rlo = gate row j, rhi = up row j of
  // the same j (tile rows 8w+gid and 64+8w+gid), so the gate is applied in registers.  Otherwise
  // 16 consecutive rows per warp.
  const int gid = lane >> 2, tq = lane & 3;
  constexpr bool gelu = GELU;
  const int rlo = gelu ? warp * 8 + gid : warp * 16 + gid;
  const int rhi = gelu ? rlo + kHalf : rlo + 8;
  const int r7 = rlo & 7;                       // == rhi & 7
  constexpr int kDwBytes = (GELU ? kHalf : 8) * 128;   // byte distance between the two rows
  constexpr int NB = MT / 8;                    // token blocks of 8 (the MMA's n)
  float* ep = reinterpret_cast<float*>(smem + (L.ep_off >= 0 ? L.ep_off : 0));
  int cslot = 0;          // ring slot and mbarrier phase of the current stage
  uint32_t cphase = 0;
  bool aborted = false;   // after a timed-out wait: skip work, keep every barrier
  for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
    Unit U;
    decode_unit<MT>(A, table, offs, u, U);
    const int nblk = (U.mt + 7) >> 3;
    float acc[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;

    for (int g = U.g0; g < U.g1; g += kGS) {
      const int slot = cslot;
      const uint32_t phase = cphase;
      if (++cslot == S) { cslot = 0; cphase ^= 1u; }
      const int gc = min(kGS, U.g1 - g);
      if (!aborted && (!mbar_wait(&full[slot], phase) || flags[0])) {
        if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
        aborted = true;
      }
      if (aborted) continue;
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(smem + slot * kCodeBytes);
      const uint8_t* xs = smem + L.x_off + slot * L.x_bytes;
      const uint8_t* ss = smem + L.sc_off + slot * L.sc_bytes;
      // scales of rows rlo / rhi for the stage's 8 groups, two bf16 per word
      uint32_t slo[4], shi[4];
      if (A.scale_mode == kScaleTma) {
        const uint4 vlo = *reinterpret_cast<const uint4*>(ss + rlo * 16);
        const uint4 vhi = *reinterpret_cast<const uint4*>(ss + rhi * 16);
        slo[0] = vlo.x; slo[1] = vlo.y; slo[2] = vlo.z; slo[3] = vlo.w;
        shi[0] = vhi.x; shi[1] = vhi.y; shi[2] = vhi.z; shi[3] = vhi.w;
      } else if (A.scale_mode == kScaleBlock) {
        // block rows hold all kg groups (kg even, g a multiple of 8: 4-byte aligned pairs)
        const uint32_t* plo = reinterpret_cast<const uint32_t*>(ss + (rlo * A.kg + g) * 2);
        const uint32_t* phi = reinterpret_cast<const uint32_t*>(ss + (rhi * A.kg + g) * 2);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          slo[p] = 2 * p < gc ? plo[p] : 0u;
          shi[p] = 2 * p < gc ? phi[p] : 0u;
        }
      } else {
        const int64_t grow_lo = tile_row_valid(A, U, rlo) ? tile_row(A, U, rlo) : tile_row(A, U, 0);
        const int64_t grow_hi = tile_row_valid(A, U, rhi) ? tile_row(A, U, rhi) : tile_row(A, U, 0);
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
      // Passes of kGP groups: dequantise rows rlo / rhi into MMA A fragments, then run the
      // token blocks.  Word (row r, group gi, quad position tq) sits at chunk gi ^ (r % 8) of the
      // 128-byte row (TMA 128-byte swizzle).  Each extracted bf16 pair is two consecutive k, so
      // k-step 0 takes elements 8tq+0..3 (x pairs .x, .y) and k-step 1 elements 8tq+4..7 (.z, .w).
      // rows rlo and rhi share the swizzle phase (rlo % 8): one address per group
      // shared address of (row rlo, chunk c, word tq) = stage + rlo*128 + ((c ^ r7) << 4) + 4 tq;
      // the stage and row bases have bits 4-6 clear, so this is base ^ (c << 4) with the r7 part
      // folded into base: one XOR per group
      const uint32_t abase = smem_u32(cw) + ((rlo * 128 + 4 * tq) ^ (r7 << 4));
      const bool mask_tail = (A.scale_mode != kScaleTma) && gc < kGS;   // TMA zero-fills past K
#pragma unroll
      for (int h = 0; h < kGS; h += kGP) {
        uint32_t fa[kGP][8];
        float fsl[kGP], fsh[kGP];
#pragma unroll
        for (int i = 0; i < kGP; ++i) {
          const int gi = h + i;
          const uint32_t aw = abase ^ static_cast<uint32_t>(gi << 4);
          const uint32_t wlo = lds32(aw);
          const uint32_t whi = lds32(aw + kDwBytes);
          // biased codes 128 + u (exact in bf16); the -136 * sum(x) term comes from one MMA per
          // k-step with the constant A = -136, so q * x = (128 + u) * x - 136 * x overall
#if W4_STREAM_BIASED
#define W4_DEQ nibbles_to_bf16x2_biased
#else
#define W4_DEQ nibbles_to_bf16x2
#endif
          fa[i][0] = W4_DEQ(wlo);        // k-step 0: elements (0,1) | (2,3)
          fa[i][1] = W4_DEQ(whi);
          fa[i][2] = W4_DEQ(wlo >> 4);
          fa[i][3] = W4_DEQ(whi >> 4);
          fa[i][4] = W4_DEQ(wlo >> 8);   // k-step 1: elements (4,5) | (6,7)
          fa[i][5] = W4_DEQ(whi >> 8);
          fa[i][6] = W4_DEQ(wlo >> 12);
          fa[i][7] = W4_DEQ(whi >> 12);
#undef W4_DEQ
          const uint32_t sl = (gi & 1) ? (slo[gi >> 1] & 0xFFFF0000u) : (slo[gi >> 1] << 16);
          const uint32_t sh = (gi & 1) ? (shi[gi >> 1] & 0xFFFF0000u) : (shi[gi >> 1] << 16);
          fsl[i] = __uint_as_float(sl);
          fsh[i] = __uint_as_float(sh);
          if (mask_tail && gi >= gc) { fsl[i] = 0.f; fsh[i] = 0.f; }   // past the K range
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < nblk) {
            const uint8_t* xrow = xs + (b * 8 + gid) * kXPitch + tq * 16;
#pragma unroll
            for (int i = 0; i < kGP; ++i) {
              const uint4 xv = *reinterpret_cast<const uint4*>(xrow + (h + i) * 64);
              const uint32_t a0[4] = {fa[i][0], fa[i][1], fa[i][2], fa[i][3]};
              const uint32_t a1[4] = {fa[i][4], fa[i][5], fa[i][6], fa[i][7]};
              float d[4];
              const float z[4] = {0.f, 0.f, 0.f, 0.f};
#if W4_STREAM_BIASED
              const uint32_t ac[4] = {kMinus136x2, kMinus136x2, kMinus136x2, kMinus136x2};
              mma_bf16_16816(d, ac, xv.x, xv.y, z);
              mma_bf16_16816(d, ac, xv.z, xv.w, d);
              mma_bf16_16816(d, a0, xv.x, xv.y, d);
#else
              mma_bf16_16816(d, a0, xv.x, xv.y, z);
#endif
              mma_bf16_16816(d, a1, xv.z, xv.w, d);
              acc[b][0] = fmaf(fsl[i], d[0], acc[b][0]);
              acc[b][1] = fmaf(fsl[i], d[1], acc[b][1]);
              acc[b][2] = fmaf(fsh[i], d[2], acc[b][2]);
              acc[b][3] = fmaf(fsh[i], d[3], acc[b][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // --------------------------- epilogue ---------------------------
    if (A.splits == 1) {
      // straight from registers: thread holds rows rlo / rhi for tokens 2tq, 2tq + 1 of each block
      if (!aborted) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < nblk) {
            const int t0 = b * 8 + 2 * tq;
            if (gelu) {
              const int Nh = A.N >> 1;
              const int j = U.nt * kHalf + warp * 8 + gid;
              if (j < Nh) {
                if (t0 < U.mt)
                  A.out[(U.r0 + t0) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][0]) * acc[b][2]);
                if (t0 + 1 < U.mt)
                  A.out[(U.r0 + t0 + 1) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][1]) * acc[b][3]);
              }
            } else {
              const int nlo = U.nt * kBN + rlo, nhi = nlo + 8;
              if (t0 < U.mt) {
                if (nlo < A.N) A.out[(U.r0 + t0) * A.N + nlo] = f32_to_bf16_bits(acc[b][0]);
                if (nhi < A.N) A.out[(U.r0 + t0) * A.N + nhi] = f32_to_bf16_bits(acc[b][2]);
              }
              if (t0 + 1 < U.mt) {
                if (nlo < A.N) A.out[(U.r0 + t0 + 1) * A.N + nlo] = f32_to_bf16_bits(acc[b][1]);
                if (nhi < A.N) A.out[(U.r0 + t0 + 1) * A.N + nhi] = f32_to_bf16_bits(acc[b][3]);
              }
            }
          }
        }
      }
      continue;
    }
    // split-K (dense, no gate): float32 partials through shared memory, then the last CTA of the
    // tile reduces them in split order
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < nblk) {
        const int t0 = b * 8 + 2 * tq;
        ep[t0 * kEpPitch + rlo] = acc[b][0];
        ep[(t0 + 1) * kEpPitch + rlo] = acc[b][1];
        ep[t0 * kEpPitch + rhi] = acc[b][2];
        ep[(t0 + 1) * kEpPitch + rhi] = acc[b][3];
      }
    }
    compute_sync();
    const int ctid = threadIdx.x;
    const int n0 = U.nt * kBN;
    if (!flags[0]) {
      for (int idx = ctid; idx < U.mt * kBN; idx += kWarps * 32) {
        const int t = idx / kBN, c = idx % kBN;
        if (n0 + c < A.N)
          A.partial[(static_cast<int64_t>(U.sp) * A.rows + U.r0 + t) * A.N + n0 + c] = ep[t * kEpPitch + c];
      }
    }
    __threadfence();
    compute_sync();
    if (ctid == 0) {
      int last = 0;
      if (!flags[0]) {
        const int tile = U.tb * A.n_tiles + U.nt;
        const int prev = atomicAdd(&A.counters[tile], 1);
        last = (prev == A.splits - 1);
        if (last) A.counters[tile] = 0;
      }
      flags[1] = last;
    }
    compute_sync();
    if (flags[1]) {
      __threadfence();
      for (int idx = ctid; idx < U.mt * kBN; idx += kWarps * 32) {
        const int t = idx / kBN, c = idx % kBN;
        if (n0 + c < A.N) {
          float sum = 0.f;
          for (int sp = 0; sp < A.splits; ++sp)
            sum += __ldcg(&A.partial[(static_cast<int64_t>(sp) * A.rows + U.r0 + t) * A.N + n0 + c]);
          A.out[(U.r0 + t) * A.N + n0 + c] = f32_to_bf16_bits(sum);
        }
      }
    }
    compute_sync();
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

// Scales [rows_total, kg] bf16 as a 2-D tensor (kg % 8 == 0): box = 8 groups x 64 rows.
static bool encode_scales_map(CUtensorMap* m, const uint16_t* scales, int64_t rows_total, int kg) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kg), static_cast<cuuint64_t>(rows_total)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kg) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(w4::kGS), static_cast<cuuint32_t>(w4::kHalf)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Ring depth and offsets for one launch: as many stages (up to kMaxStages) as fit the per-CTA
// shared-memory budget next to the fixed parts.
static w4::Layout make_layout(int MT, int scale_mode, int kg, int E, bool split) {
  w4::Layout L{};
  L.x_bytes = MT * w4::kXPitch;
  L.sc_bytes = scale_mode == w4::kScaleTma ? 2 * w4::kHalf * w4::kGS * 2
             : scale_mode == w4::kScaleBlock ? 2 * w4::kHalf * kg * 2 : 16;
  L.sc_bytes = (L.sc_bytes + 127) & ~127;
  const int ep_bytes = split ? MT * w4::kEpPitch * 4 : 0;
  const int fixed = ep_bytes + 2 * w4::kMaxStages * 8 + 16 + (E + 1) * 8 + 1024;   // + alignment slack
  const int per_stage = w4::kCodeBytes + L.x_bytes + L.sc_bytes;
  int S = (w4::kSmemPerCta - fixed) / per_stage;
  if (S > w4::kMaxStages) S = w4::kMaxStages;
  L.stages = S;
  L.x_off = S * w4::kCodeBytes;
  L.sc_off = L.x_off + S * L.x_bytes;
  int off = L.sc_off + S * L.sc_bytes;
  L.ep_off = split ? off : -1;
  off += ep_bytes;
  L.bar_off = (off + 7) & ~7;
  off = L.bar_off + 2 * S * 8;
  L.flag_off = off;
  off += 16;
  L.table_off = off;
  off += (E + 1) * 8;
  L.total = off + 1024;
  return L;
}

struct StreamPlan {
  int splits, stages_per_split, n_tiles, MT;
};

static StreamPlan plan_stream(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  StreamPlan p;
  const int kg = K / 32;
  const int kstages = (kg + w4::kGS - 1) / w4::kGS;
  // token block: 8 rows when experts hold few rows on average (keeps the activation ring small and
  // the weight ring deep), else 16
  p.MT = (rows <= 6LL * E) ? 8 : 16;
  p.n_tiles = (epi == W4_EPI_GELU_GATE) ? ((N / 2) + w4::kHalf - 1) / w4::kHalf
                                        : (N + w4::kBN - 1) / w4::kBN;
  p.splits = 1;
  if (dense) {
    // split K while the units do not fill the CTAs four times over and the float32 partials
    // stay below ~1/8 of the weight bytes
    const int64_t ntb = (rows + p.MT - 1) / p.MT;
    const double wbytes = static_cast<double>(N) * K * 0.5625;
    while (p.splits * 2 <= kstages && ntb * p.n_tiles * p.splits < 4LL * w4::kCtasPerSm * sm_count &&
           static_cast<double>(p.splits * 2) * rows * N * 8.0 <= wbytes / 8.0)
      p.splits *= 2;
  }
  p.stages_per_split = (kstages + p.splits - 1) / p.splits;
  p.splits = (kstages + p.stages_per_split - 1) / p.stages_per_split;
  return p;
}

// Split-K workspace: the per-tile arrival counters first (cleared by every launch), then the
// float32 partials [splits, rows, N].
static size_t counters_bytes(const StreamPlan& p, int64_t rows) {
  const int64_t ntb = (rows + p.MT - 1) / p.MT;
  return (static_cast<size_t>(ntb * p.n_tiles) * sizeof(int32_t) + 255) & ~size_t(255);
}

size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  if (p.splits == 1) return 0;
  return counters_bytes(p, rows) + static_cast<size_t>(p.splits) * rows * N * sizeof(float);
}

template <int MT, bool GELU>
static w4_status launch_mt(const CUtensorMap& tmap, const CUtensorMap& smap, const w4::StreamArgs& A,
                           int sm_count, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel<MT, GELU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             w4::kSmemPerCta) != cudaSuccess)
      return W4_ERR_CUDA;
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel<MT, GELU>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  w4::stream_gemm_kernel<MT, GELU><<<sm_count * w4::kCtasPerSm, w4::kThreads, A.L.total, stream>>>(tmap, smap, A);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
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
  A.dev_status = dev_status;
  // Scale staging: 2-D TMA when a scale row is a whole number of 16-byte chunks; else the tile's
  // contiguous 64-row scale blocks by bulk copy when they are 16-byte aligned and small; else
  // direct loads.
  const bool s16 = (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
  if (A.kg % 8 == 0 && s16) {
    A.scale_mode = w4::kScaleTma;
  } else if (p.splits == 1 && A.kg % 2 == 0 && A.kg <= w4::kBlockMaxKg && N % 8 == 0 && s16 &&
             (epi == W4_EPI_GELU_GATE ? (N / 2) % w4::kHalf == 0 : N % w4::kBN == 0)) {
    // (whole tiles only: the 64-row blocks are plain bulk copies and must stay inside the array)
    A.scale_mode = w4::kScaleBlock;
  } else {
    A.scale_mode = w4::kScaleLdg;
  }
  A.L = make_layout(p.MT, A.scale_mode, A.kg, E, p.splits > 1);
  if (A.L.stages < 2) return W4_ERR_UNSUPPORTED;
  if (p.splits > 1) {
    const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count);
    if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
    const size_t cb = counters_bytes(p, rows);
    A.counters = static_cast<int32_t*>(ws);
    A.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + cb);
    // the arrival counters must start at zero whatever the workspace held before
    if (rows > 0 && cudaMemsetAsync(ws, 0, cb, stream) != cudaSuccess) return W4_ERR_CUDA;
  }
  if (rows == 0) return W4_OK;
  CUtensorMap tmap, smap;
  std::memset(&smap, 0, sizeof(smap));
  if (!encode_codes_map(&tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  if (A.scale_mode == w4::kScaleTma &&
      !encode_scales_map(&smap, scales, static_cast<int64_t>(E) * N, A.kg))
    return W4_ERR_CUDA;
  const bool gelu = A.epi == W4_EPI_GELU_GATE;
  if (p.MT == 8)
    return gelu ? launch_mt<8, true>(tmap, smap, A, sm_count, stream)
                : launch_mt<8, false>(tmap, smap, A, sm_count, stream);
  return gelu ? launch_mt<16, true>(tmap, smap, A, sm_count, stream)
              : launch_mt<16, false>(tmap, smap, A, sm_count, stream);
}
