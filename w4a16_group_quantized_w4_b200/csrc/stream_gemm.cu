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
//   * Work unit = (expert e, block of <= 16 routed rows, tile of 128 weight rows, K split).  A
//     persistent grid (two CTAs per SM) walks the units; the unit table is a prefix sum over the
//     experts built on the device from expert_offsets, so no host synchronisation is needed.
//   * A 3-stage shared-memory ring per CTA (6 stages in flight per SM).  One stage = 8 groups
//     (256 k) of the 128-row code tile (two 64-row 2-D TMA boxes, 128-byte swizzle), the matching
//     bf16 scales (two 2-D TMA boxes when the scale row pitch is 16-byte aligned, else the tile's
//     contiguous 64-row scale blocks by 1-D bulk copy), and the <= 16 activation rows gathered by
//     a_row_of_pair (1-D bulk copies).  Everything completes on the stage's mbarrier.  Lane 0 of
//     warp 0 issues the copies one ring-length ahead of the math.
//   * Eight warps each own 16 weight rows.  A thread's 32-bit code word becomes four bf16 pairs
//     (one lop3 + one packed fma per pair), which are exactly the A fragments of two m16n8k16
//     MMAs with the tokens as the n = 8 side.  The packed nibble order puts two consecutive k in
//     each extracted pair, so the activation B fragments are plain 16-byte shared loads.  Each
//     group's MMAs start from zero and the group's scale is folded in with one fp32 FMA per
//     accumulator: acc += s_g * (sum over the group of q * x).  Products q * x are exact in fp32.
//   * Epilogue from registers, without a CTA barrier: with the GELU gate each warp's two A-fragment
//     row sets are 8 gate rows and the 8 up rows of the same outputs, so h = gelu(g) * u is formed
//     in the thread that holds both.  Dense split-K writes float32 partials that the last CTA of
//     the tile reduces in a fixed order (deterministic).
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"

namespace w4 {

constexpr int kStages = 3;
constexpr int kGS = 8;                        // groups per stage
constexpr int kWarps = 8;                     // all warps compute; warp 0 also issues the copies
constexpr int kThreads = kWarps * 32;
constexpr int kBN = 16 * kWarps;              // weight rows per tile
constexpr int kHalf = kBN / 2;                // rows per TMA box
constexpr int kMT = 16;                       // routed rows (tokens) per unit
constexpr int kXPitch = kGS * 64 + 64;        // bytes per token row in an activation stage
constexpr int kCodeBytes = kBN * kGS * 16;    // 16 KB
constexpr int kXBytes = kMT * kXPitch;        // 9 KB
constexpr int kBlockMaxKg = 24;               // scale-block mode: two 64-row blocks of <= 24 groups
constexpr int kScaleBytes = 2 * kHalf * kBlockMaxKg * 2;   // 6 KB
constexpr int kEpPitch = kBN + 4;             // floats per token row in the epilogue buffer
constexpr int kCtasPerSm = 2;

enum ScaleMode { kScaleLdg = 0, kScaleBlock = 1, kScaleTma = 2 };

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

// Source row in `a` of routed row r (checked; out-of-range indices read row 0 and are reported).
__device__ __forceinline__ int64_t gather_row(const StreamArgs& A, int64_t r) {
  int64_t src = A.a_row_of_pair ? static_cast<int64_t>(__ldg(A.a_row_of_pair + r) / A.k_div) : r;
  if (src < 0 || src >= A.a_rows) {
    set_status(A.dev_status, W4_ERR_INVALID_ARG);
    src = 0;
  }
  return src;
}

// The copy side of the ring: a cursor over (unit, stage) that runs kStages - 1 stages ahead.
struct Producer {
  int64_t u;
  Unit U;
  int g;
  int64_t src_row;
  bool done;
};

__device__ __forceinline__ void producer_load_unit(const StreamArgs& A, const int* table, const int* offs,
                                                   int64_t total, Producer& P, int lane) {
  P.done = P.u >= total;
  if (P.done) return;
  decode_unit(A, table, offs, P.u, P.U);
  P.g = P.U.g0;
  P.src_row = lane < P.U.mt ? gather_row(A, P.U.r0 + lane) : 0;
}

// Issues the stage under the cursor into its ring slot (warp-wide call) and advances the
// cursor.  Returns false if the bounded wait for the slot gave up.
__device__ __forceinline__ bool producer_issue(const StreamArgs& A, const CUtensorMap* tm_codes,
                                               const CUtensorMap* tm_scales, uint8_t* smem,
                                               uint64_t* full, uint64_t* empty, const int* table,
                                               const int* offs, int64_t total, Producer& P,
                                               uint32_t stage_index, int lane) {
  if (P.done) return true;
  const int slot = stage_index % kStages;
  const uint32_t round = stage_index / kStages;
  if (round > 0) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(&empty[slot], (round - 1) & 1);
    if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
  }
  const Unit& U = P.U;
  const int g = P.g;
  const int gc = min(kGS, U.g1 - g);
  uint8_t* cdst = smem + SmemLayout::codes + slot * kCodeBytes;
  uint8_t* xdst = smem + SmemLayout::x + slot * kXBytes;
  uint8_t* sdst = smem + SmemLayout::sc + slot * kScaleBytes;
  const uint32_t xbytes = static_cast<uint32_t>(gc) * 64u;
  if (lane == 0) {
    const int64_t row_a = tile_row(A, U, 0);
    const int64_t row_b = tile_row(A, U, kHalf);
    uint32_t sbytes = 0;
    if (A.scale_mode == kScaleTma) sbytes = 2 * kHalf * kGS * 2;
    else if (A.scale_mode == kScaleBlock) sbytes = 2 * kHalf * A.kg * 2;
    mbar_arrive_expect_tx(&full[slot], kCodeBytes + sbytes + xbytes * U.mt);
    tma_load_2d(cdst, tm_codes, g * 4, static_cast<int32_t>(row_a), &full[slot]);
    tma_load_2d(cdst + kHalf * 128, tm_codes, g * 4, static_cast<int32_t>(row_b), &full[slot]);
    if (A.scale_mode == kScaleTma) {
      tma_load_2d(sdst, tm_scales, g, static_cast<int32_t>(row_a), &full[slot]);
      tma_load_2d(sdst + kHalf * kGS * 2, tm_scales, g, static_cast<int32_t>(row_b), &full[slot]);
    } else if (A.scale_mode == kScaleBlock) {
      const uint32_t blk = kHalf * A.kg * 2;
      bulk_g2s(sdst, A.scales + row_a * A.kg, blk, &full[slot]);
      bulk_g2s(sdst + blk, A.scales + row_b * A.kg, blk, &full[slot]);
    }
  }
  __syncwarp();
  if (lane < U.mt)
    bulk_g2s(xdst + lane * kXPitch, A.a + P.src_row * A.K + static_cast<int64_t>(g) * 32, xbytes,
             &full[slot]);
  P.g += kGS;
  if (P.g >= U.g1) {
    P.u += gridDim.x;
    producer_load_unit(A, table, offs, total, P, lane);
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, StreamArgs A) {
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
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t total_units = table[A.E];

  Producer P;
  uint32_t issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmap_codes);
      if (A.scale_mode == kScaleTma) prefetch_tmap(&tmap_scales);
    }
    P.u = blockIdx.x;
    producer_load_unit(A, table, offs, total_units, P, lane);
    for (; issued < kStages - 1 && !P.done; ++issued)
      producer_issue(A, &tmap_codes, &tmap_scales, smem, full, empty, table, offs, total_units, P,
                     issued, lane);
  }

  // Rows of this thread's two A-fragment rows.  GELU gate: rlo = gate row j, rhi = up row j of
  // the same j (tile rows 8w+gid and 64+8w+gid), so the gate is applied in registers.  Otherwise
  // 16 consecutive rows per warp.
  const int gid = lane >> 2, tq = lane & 3;
  const bool gelu = (A.epi == W4_EPI_GELU_GATE);
  const int rlo = gelu ? warp * 8 + gid : warp * 16 + gid;
  const int rhi = gelu ? rlo + kHalf : rlo + 8;
  const int r7 = rlo & 7;                       // == rhi & 7
  const int dw = (rhi - rlo) * 32;              // word distance between the two rows
  float* ep = reinterpret_cast<float*>(smem + SmemLayout::ep);
  uint32_t it = 0;
  bool aborted = false;   // after a timed-out wait: skip work, keep every barrier
  for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
    Unit U;
    decode_unit(A, table, offs, u, U);
    const int nblk = (U.mt + 7) >> 3;
    float acc[2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;

    for (int g = U.g0; g < U.g1; g += kGS, ++it) {
      // keep the ring full: warp 0 issues the stage kStages - 1 ahead of this one
      if (warp == 0 && !aborted && !P.done) {
        if (!producer_issue(A, &tmap_codes, &tmap_scales, smem, full, empty, table, offs,
                            total_units, P, issued, lane)) {
          if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
          aborted = true;
        }
        ++issued;
      }
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
      const uint8_t* ss = smem + SmemLayout::sc + slot * kScaleBytes;
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
      // Two halves of 4 groups: dequantise rows rlo / rhi into MMA A fragments, then run the
      // token blocks.  Word (row r, group gi, quad position tq) sits at chunk gi ^ (r % 8) of the
      // 128-byte row (TMA 128-byte swizzle).  Each extracted bf16 pair is two consecutive k, so
      // k-step 0 takes elements 8tq+0..3 (x pairs .x, .y) and k-step 1 elements 8tq+4..7 (.z, .w).
      // rows rlo and rhi share the swizzle phase (rlo % 8): one address per group
      const uint32_t* cwl = cw + rlo * 32 + tq;
      const bool mask_tail = (A.scale_mode != kScaleTma) && gc < kGS;   // TMA zero-fills past K
#pragma unroll
      for (int h = 0; h < kGS; h += 4) {
        uint32_t fa[4][8];
        float fsl[4], fsh[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int gi = h + i;
          const uint32_t* pw = cwl + ((gi ^ r7) << 2);
          const uint32_t wlo = pw[0];
          const uint32_t whi = pw[dw];
          fa[i][0] = nibbles_to_bf16x2(wlo);        // k-step 0: elements (0,1) | (2,3)
          fa[i][1] = nibbles_to_bf16x2(whi);
          fa[i][2] = nibbles_to_bf16x2(wlo >> 4);
          fa[i][3] = nibbles_to_bf16x2(whi >> 4);
          fa[i][4] = nibbles_to_bf16x2(wlo >> 8);   // k-step 1: elements (4,5) | (6,7)
          fa[i][5] = nibbles_to_bf16x2(whi >> 8);
          fa[i][6] = nibbles_to_bf16x2(wlo >> 12);
          fa[i][7] = nibbles_to_bf16x2(whi >> 12);
          const uint32_t sl = (gi & 1) ? (slo[gi >> 1] & 0xFFFF0000u) : (slo[gi >> 1] << 16);
          const uint32_t sh = (gi & 1) ? (shi[gi >> 1] & 0xFFFF0000u) : (shi[gi >> 1] << 16);
          fsl[i] = __uint_as_float(sl);
          fsh[i] = __uint_as_float(sh);
          if (mask_tail && gi >= gc) { fsl[i] = 0.f; fsh[i] = 0.f; }   // past the K range
        }
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (b < nblk) {
            const uint8_t* xrow = xs + (b * 8 + gid) * kXPitch + tq * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 xv = *reinterpret_cast<const uint4*>(xrow + (h + i) * 64);
              const uint32_t a0[4] = {fa[i][0], fa[i][1], fa[i][2], fa[i][3]};
              const uint32_t a1[4] = {fa[i][4], fa[i][5], fa[i][6], fa[i][7]};
              float d[4];
              const float z[4] = {0.f, 0.f, 0.f, 0.f};
              mma_bf16_16816(d, a0, xv.x, xv.y, z);
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
        for (int b = 0; b < 2; ++b) {
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
    for (int b = 0; b < 2; ++b) {
      if (b < nblk) {
        const int t0 = b * 8 + 2 * tq;
        ep[t0 * kEpPitch + rlo] = acc[b][0];
        ep[(t0 + 1) * kEpPitch + rlo] = acc[b][1];
        ep[t0 * kEpPitch + rhi] = acc[b][2];
        ep[(t0 + 1) * kEpPitch + rhi] = acc[b][3];
      }
    }
    __syncthreads();
    const int ctid = threadIdx.x;
    const int n0 = U.nt * kBN;
    if (!flags[0]) {
      for (int idx = ctid; idx < U.mt * kBN; idx += kThreads) {
        const int t = idx / kBN, c = idx % kBN;
        if (n0 + c < A.N)
          A.partial[(static_cast<int64_t>(U.sp) * A.rows + U.r0 + t) * A.N + n0 + c] = ep[t * kEpPitch + c];
      }
    }
    __threadfence();
    __syncthreads();
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
    __syncthreads();
    if (flags[1]) {
      __threadfence();
      for (int idx = ctid; idx < U.mt * kBN; idx += kThreads) {
        const int t = idx / kBN, c = idx % kBN;
        if (n0 + c < A.N) {
          float sum = 0.f;
          for (int sp = 0; sp < A.splits; ++sp)
            sum += __ldcg(&A.partial[(static_cast<int64_t>(sp) * A.rows + U.r0 + t) * A.N + n0 + c]);
          A.out[(U.r0 + t) * A.N + n0 + c] = f32_to_bf16_bits(sum);
        }
      }
    }
    __syncthreads();
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
    // split K while the units do not fill the CTAs four times over and the float32 partials
    // stay below ~1/8 of the weight bytes
    const int64_t ntb = (rows + w4::kMT - 1) / w4::kMT;
    const double wbytes = static_cast<double>(N) * K * 0.5625;
    while (p.splits * 2 <= kstages && ntb * p.n_tiles * p.splits < 4LL * w4::kCtasPerSm * sm_count &&
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
  if (p.splits > 1) {
    const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count);
    if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
    size_t pb = static_cast<size_t>(p.splits) * rows * N * sizeof(float);
    pb = (pb + 255) & ~size_t(255);
    A.partial = static_cast<float*>(ws);
    A.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + pb);
  }
  if (rows == 0) return W4_OK;
  CUtensorMap tmap, smap;
  std::memset(&smap, 0, sizeof(smap));
  if (!encode_codes_map(&tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  if (A.scale_mode == w4::kScaleTma &&
      !encode_scales_map(&smap, scales, static_cast<int64_t>(E) * N, A.kg))
    return W4_ERR_CUDA;
  const size_t smem = stream_smem_bytes(E);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(stream_smem_bytes(1024))) != cudaSuccess)
      return W4_ERR_CUDA;
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  w4::stream_gemm_kernel<<<sm_count * w4::kCtasPerSm, w4::kThreads, smem, stream>>>(tmap, smap, A);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
