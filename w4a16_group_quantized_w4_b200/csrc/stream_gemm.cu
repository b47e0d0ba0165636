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
//   * A preparation pass (one warp per routed row) writes each activation row once, gathered into
//     routed-row order, as fp16 with a power-of-two exponent per row: x' = x * 2^f, f putting the
//     row's largest |x| in [2^14, 2^15), with the multiplier 2^-f beside every 256-k block.
//     Within every 8 consecutive k the elements 2, 3, 6, 7 are stored divided by 16 (see the
//     dequantisation below).  Next to each 256-k block of a row it stores the block's 8 group
//     corrections
//     c = -(1032 * sum of x' over elements 0, 1, 4, 5 + 1152 * sum of the stored x'/16 values),
//     as quads {c(r), c(r + 1), c(r), c(r + 1)} for the row pair (r, r + 1).
//   * Work unit = (expert e, block of <= MT routed rows (MT = 8 or 16), tile of 128 weight rows,
//     K split).  A persistent grid (two CTAs per SM) walks the units; the unit table is a prefix
//     sum over the experts built on the device from expert_offsets (no host synchronisation).
//   * Each CTA = 8 compute warps + 1 producer warp.  The producer keeps a shared-memory ring as
//     deep as the per-CTA shared-memory budget allows full: one stage = 8 groups (256 k) of the
//     128-row code tile (two 64-row 2-D TMA boxes, 128-byte swizzle), the matching bf16 scales
//     (two 2-D TMA boxes when a scale row is a whole number of 16-byte chunks, else the tile's
//     contiguous 64-row scale blocks by 1-D bulk copy), and the prepared activation rows and
//     correction quads (1-D bulk copies).  Everything completes on the stage's mbarrier.
//   * A compute warp owns 16 weight rows.  A thread's 32-bit code word gives its four fp16 pairs
//     with one shift and four lop3: fields at bits 0..3 / 16..19 become 1024 + u, fields at bits
//     4..7 / 20..23 become 1024 + 16 u (exact), and the activations at those positions were
//     stored divided by 16, so every product is (bias + u) * x' with bias 1024 or 64 (in units
//     of x').  The group's correction quad is the C operand of its first MMA, which removes the
//     bias and the -8 of q = u - 8: d = sum over the group of q * x'.  The packed nibble order
//     puts two consecutive k in each extracted pair, so the activation B fragments are plain
//     16-byte shared loads.  The group's scale is folded in with one fp32 FMA per accumulator:
//     acc += s_g * d.  The epilogue multiplies by the token's 2^-f, read from the unit's last
//     stage (a global load there would wait behind the weight stream).
//   * Epilogue from registers, without a CTA barrier: with the GELU gate each warp's two A-fragment
//     row sets are 8 gate rows and the 8 up rows of the same outputs, so h = gelu(g) * u is formed
//     in the thread that holds both.  When the units would not cover the pipelines (dense GEMVs,
//     grouped calls with a few routed rows, e.g. one decode token through 8 experts), K is split:
//     float32 partials that the last pipeline of the tile reduces in a fixed order
//     (deterministic), applying the GELU gate after the sum.
// Rounding: the products are exact; each MMA sums 16 products of up to (1024 + 240) * 2^15 in
// float32 next to the bias, which the correction cancels, so a group's sum carries an absolute
// error of a few float32 units of its bias term (about 2^-13 of the group's mean |x'| times the
// group size), far inside the bf16 rounding of the output.
#include <cudaTypedefs.h>

#include <cstring>

#include <cuda_fp16.h>

#include "common.cuh"

namespace w4 {

#ifndef W4_STREAM_GROUPS_PER_PASS
#define W4_STREAM_GROUPS_PER_PASS 4           // groups dequantised into registers at a time
#endif

constexpr int kMaxStages = 6;
constexpr int kGS = 8;                        // groups per stage
constexpr int kGP = W4_STREAM_GROUPS_PER_PASS;
constexpr int kWarps = 8;                     // compute warps per pipeline
constexpr int kPipes = 2;                     // pipelines per CTA (one CTA per SM)
constexpr int kPipeWarps = kWarps + 1;        // + one producer warp
constexpr int kThreads = kPipes * kPipeWarps * 32;
constexpr int kBN = 16 * kWarps;              // weight rows per tile
constexpr int kHalf = kBN / 2;                // rows per TMA box
constexpr int kXPitch = kGS * 64 + 64;        // bytes per token row in an activation stage
constexpr int kXBlock = kGS * 64;             // prepared activation bytes per row and stage
constexpr int kXCopy = kXBlock + 16;          // + the row's multiplier 2^-f (and 12 spare bytes)
constexpr int kQBlock = kGS * 16;             // correction-quad bytes per row and stage
constexpr int kPrepStage = kXCopy + kQBlock;  // prepared bytes per row and 256-k block (656)
constexpr int kQPitch = kQBlock + 16;         // bytes per row pair in a stage's quad area
constexpr int kCodeBytes = kBN * kGS * 16;    // 16 KB
constexpr int kBlockMaxKg = 24;               // scale-block mode: two 64-row blocks of <= 24 groups
constexpr int kEpPitch = kBN + 4;             // floats per token row in the epilogue buffer
constexpr int kDescBytes = 32;                // stage descriptor
constexpr int kPB = 12;                       // preparation pass: 256-k blocks per register batch
// dynamic shared memory of the CTA (227 KB opt-in limit per block)
constexpr int kSmemPerCta = 232448;

enum ScaleMode { kScaleLdg = 0, kScaleBlock = 1, kScaleTma = 2 };

// Shared-memory layout of one pipeline, fixed per launch (offsets from the pipeline's
// 1024-byte aligned base); the two pipelines' regions follow each other, then the unit table.
struct Layout {
  int stages;
  int x_off, x_bytes;        // activation ring: stages x (MT rows x kXPitch)
  int q_off, q_bytes;        // correction quads: stages x (MT/2 row pairs x kQPitch)
  int sc_off, sc_bytes;      // scale ring: stages x sc_bytes
  int desc_off;              // stages x kDescBytes stage descriptors
  int ep_off;                // split-K epilogue buffer (MT x kEpPitch floats), or -1
  int bar_off;               // 2 * stages mbarriers, then the epilogue barrier
  int flag_off;              // 16 bytes
  int pipe_bytes;            // one pipeline's region (multiple of 1024)
  int table_off;             // int table[E + 1], int offs[E + 1] (shared)
  int total;
};

struct StreamArgs {
  const uint8_t* xw;        // prepared rows: [rows][kstages][656 bytes] (fp16 x', 2^-f, quads)
  int64_t xw_stride;        // bytes per prepared row
  const uint16_t* scales;   // [E*N, kg]
  const int32_t* offsets;   // [E+1] or null (one expert with `rows` rows)
  int E, N, K, kg;
  int64_t rows;
  int epi;
  uint16_t* out;
  float* partial;           // [splits, rows, N] (splits > 1)
  int32_t* counters;        // [tiles] (splits > 1)
  int splits, stages_per_split, n_tiles;
  int pf_all;               // prefetch every stage of the pipeline's units into L2 at the start
  Layout L;
  int32_t* dev_status;
};

struct Unit {
  int e, tb, nt, sp;
  int64_t r0;
  int mt;
  int g0, g1;
  int tile;               // dense id of (e, tb, nt)
};

// Stage descriptor written by the producer next to the stage's data, read by the compute warps
// after the stage's full barrier: the unit the stage belongs to and where it sits in it.
enum : int { kDescFirst = 1, kDescLast = 2, kDescDone = 4 };
// {r0, first group, weight tile, mt | groups << 5 | flags << 9} in the first 16 bytes (read every
// stage), {expert, K split, tile id, 0} in the second (read only by the split-K epilogue and the
// direct-load scale mode).  The tile id numbers the (expert, token block, weight tile) triples
// 0.. densely; the split-K arrival counters are indexed by it.
struct __align__(16) StageDesc {
  int r0;
  int g;
  int nt;
  int bits;
  int e, sp, tile, pad;
};
__device__ __forceinline__ int desc_mt(const StageDesc& d) { return d.bits & 31; }
__device__ __forceinline__ int desc_gc(const StageDesc& d) { return (d.bits >> 5) & 15; }
__device__ __forceinline__ int desc_flags(const StageDesc& d) { return (d.bits >> 9) & 7; }

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
  U.tile = table[U.e] / A.splits + U.tb + ntb * U.nt;
  U.g0 = U.sp * A.stages_per_split * kGS;
  U.g1 = min(A.kg, U.g0 + A.stages_per_split * kGS);
}

// global weight row (e*N + n) of tile row r in [0, kBN)
__device__ __forceinline__ int64_t tile_row(const StreamArgs& A, int e, int nt, int r) {
  int n;
  if (A.epi == W4_EPI_GELU_GATE) {
    const int j = nt * kHalf + (r & (kHalf - 1));
    n = (r < kHalf) ? j : (A.N >> 1) + j;
  } else {
    n = nt * kBN + r;
  }
  return static_cast<int64_t>(e) * A.N + n;
}

__device__ __forceinline__ bool tile_row_valid(const StreamArgs& A, int nt, int r) {
  if (A.epi == W4_EPI_GELU_GATE) return nt * kHalf + (r & (kHalf - 1)) < (A.N >> 1);
  return nt * kBN + r < A.N;
}


// One k-step of a group: the four fp16 pairs of code words wl (row rlo) and wh (row rhi) --
// fields at bits 0..3 / 16..19 as 1024 + u, at bits 4..7 / 20..23 as 1024 + 16 u -- times the
// activation pair (b0, b1), plus c.  The extraction sits in the same asm block as the MMA so the
// fragment registers live only across it.
// The exponent pattern 0x64006400 comes in as a register (one immediate per lop3).
__device__ __forceinline__ void mma_nib(float (&d)[4], uint32_t wl, uint32_t wh, uint32_t b0, uint32_t b1,
                                        const float (&c)[4], uint32_t e1024) {
  asm("{\n .reg .b32 a0, a1, a2, a3;\n"
      " lop3.b32 a0, %4, 0x000F000F, %12, 0xEA;\n"
      " lop3.b32 a1, %5, 0x000F000F, %12, 0xEA;\n"
      " lop3.b32 a2, %4, 0x00F000F0, %12, 0xEA;\n"
      " lop3.b32 a3, %5, 0x00F000F0, %12, 0xEA;\n"
      " mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {a0,a1,a2,a3}, {%6,%7},"
      " {%8,%9,%10,%11};\n}\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(wl), "r"(wh), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]), "r"(e1024));
}

template <int MT, bool GELU, int SCALE>
__global__ void __launch_bounds__(kThreads, 1)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, StreamArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (128-byte swizzle atoms), derived by pointer arithmetic so that every
  // pointer below stays in the shared address space (plain shared loads, not generic ones)
  uint8_t* smem0 = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Layout& L = A.L;
  const int S = L.stages;
  const int warp_all = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // warps 0..7: pipeline 0 compute, 8..15: pipeline 1 compute, 16 / 17: their producers
  const bool is_producer = warp_all >= kPipes * kWarps;
  const int pipe = is_producer ? warp_all - kPipes * kWarps : warp_all / kWarps;
  const int warp = is_producer ? kWarps : warp_all % kWarps;
  uint8_t* smem = smem0 + pipe * L.pipe_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + S;
  uint64_t* epi_bar = empty + S;     // split-K epilogue: the pipeline's compute warps meet here
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L.flag_off);
  StageDesc* desc = reinterpret_cast<StageDesc*>(smem + L.desc_off);
  int* table = reinterpret_cast<int*>(smem0 + L.table_off);
  int* offs = table + (A.E + 1);

  // Activation and quad stages start zeroed: token columns past a block's rows then read finite
  // values (their results are dropped).  The activation and quad areas are contiguous.  This
  // set-up overlaps the end of the previous kernel on the stream; global memory waits for it.
  // (No early trigger here: kernels after the GEMM launch when it completes.)
  for (int p = 0; p < kPipes; ++p)
    for (int i = threadIdx.x; i < S * (L.x_bytes + L.q_bytes) / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem0 + p * L.pipe_bytes + L.x_off)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();

  // unit table: table[e] = first unit of expert e, table[E] = total; offsets copied to offs[].
  // Offsets that are not non-decreasing from 0 to rows make the launch a no-op (W4_ERR_INVALID_ARG).
  if (warp_all == 0) {
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
  if (is_producer && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    mbar_init(epi_bar, kWarps);
    flags[0] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t total_units = table[A.E];
  const int64_t vb = static_cast<int64_t>(blockIdx.x) * kPipes + pipe;   // this pipeline's id
  const int64_t nvb = static_cast<int64_t>(gridDim.x) * kPipes;

  if (is_producer) {
    // ------------------------------- producer -------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_codes);
      if (SCALE == kScaleTma) prefetch_tmap(&tmap_scales);
    }
    int slot = 0;
    uint32_t phase = 0;        // phase of the empty barrier to wait for on the next lap
    bool first_lap = true;
    // claims the next ring slot (false: a wait timed out or the compute warps gave up)
    auto claim = [&]() -> bool {
      if (!first_lap) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_ring(&empty[slot], phase);
        if (!__shfl_sync(0xffffffffu, ok, 0) || flags[0]) {
          if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
          return false;
        }
      }
      return true;
    };
    auto advance = [&]() { if (++slot == S) { slot = 0; if (!first_lap) phase ^= 1u; first_lap = false; } };
    if (A.pf_all && lane == 0) {
      // weights that fit in L2 several times over: ask for all of this pipeline's code and scale
      // tiles now, so DRAM streams them at full rate while the ring fills from L2
      for (int64_t u = vb; u < total_units; u += nvb) {
        Unit U;
        decode_unit<MT>(A, table, offs, u, U);
        const int32_t ra = static_cast<int32_t>(tile_row(A, U.e, U.nt, 0));
        const int32_t rb = static_cast<int32_t>(tile_row(A, U.e, U.nt, kHalf));
        for (int g = U.g0; g < U.g1; g += kGS) {
          tma_prefetch_2d(&tmap_codes, g * 4, ra);
          tma_prefetch_2d(&tmap_codes, g * 4, rb);
          if (SCALE == kScaleTma) {
            tma_prefetch_2d(&tmap_scales, g, ra);
            tma_prefetch_2d(&tmap_scales, g, rb);
          }
        }
        if (SCALE == kScaleBlock) {
          bulk_prefetch_l2(A.scales + static_cast<int64_t>(ra) * A.kg, kHalf * A.kg * 2);
          bulk_prefetch_l2(A.scales + static_cast<int64_t>(rb) * A.kg, kHalf * A.kg * 2);
        }
      }
    }
    for (int64_t u = vb; u < total_units; u += nvb) {
      Unit U;
      decode_unit<MT>(A, table, offs, u, U);
      const uint8_t* xsrc = A.xw + (U.r0 + (lane < U.mt ? lane : 0)) * A.xw_stride;
      const int64_t row_a = tile_row(A, U.e, U.nt, 0);
      const int64_t row_b = tile_row(A, U.e, U.nt, kHalf);
      for (int g = U.g0; g < U.g1; g += kGS) {
        if (!claim()) return;
        uint8_t* cdst = smem + slot * kCodeBytes;
        uint8_t* xdst = smem + L.x_off + slot * L.x_bytes;
        uint8_t* qdst = smem + L.q_off + slot * L.q_bytes;
        uint8_t* sdst = smem + L.sc_off + slot * L.sc_bytes;
        if (lane == 0) {
          StageDesc dsc;
          dsc.r0 = static_cast<int>(U.r0);
          dsc.g = g;
          dsc.nt = U.nt;
          const int fl = (g == U.g0 ? kDescFirst : 0) | (g + kGS >= U.g1 ? kDescLast : 0);
          dsc.bits = U.mt | (min(kGS, U.g1 - g) << 5) | (fl << 9);
          dsc.e = U.e;
          dsc.sp = U.sp;
          dsc.tile = U.tile;
          dsc.pad = 0;
          desc[slot] = dsc;
          uint32_t sbytes = 0;
          if (SCALE == kScaleTma) sbytes = 2 * kHalf * kGS * 2;
          else if (SCALE == kScaleBlock) sbytes = 2 * kHalf * A.kg * 2;
          // whole 256-k blocks of every row (the preparation pass zero-fills past K) and the
          // quads of the even rows; the arrive releases the descriptor written above
          mbar_arrive_expect_tx(&full[slot], kCodeBytes + sbytes + kXCopy * U.mt + kQBlock * ((U.mt + 1) >> 1));
          tma_load_2d(cdst, &tmap_codes, g * 4, static_cast<int32_t>(row_a), &full[slot]);
          tma_load_2d(cdst + kHalf * 128, &tmap_codes, g * 4, static_cast<int32_t>(row_b), &full[slot]);
          if (SCALE == kScaleTma) {
            tma_load_2d(sdst, &tmap_scales, g, static_cast<int32_t>(row_a), &full[slot]);
            tma_load_2d(sdst + kHalf * kGS * 2, &tmap_scales, g, static_cast<int32_t>(row_b), &full[slot]);
          } else if (SCALE == kScaleBlock) {
            const uint32_t blk = kHalf * A.kg * 2;
            bulk_g2s(sdst, A.scales + row_a * A.kg, blk, &full[slot]);
            bulk_g2s(sdst + blk, A.scales + row_b * A.kg, blk, &full[slot]);
          }
        }
        __syncwarp();
        if (lane < U.mt) {
          const uint8_t* blk = xsrc + static_cast<int64_t>(g / kGS) * kPrepStage;
          bulk_g2s(xdst + lane * kXPitch, blk, kXCopy, &full[slot]);
          if (!(lane & 1)) bulk_g2s(qdst + (lane >> 1) * kQPitch, blk + kXCopy, kQBlock, &full[slot]);
        }
        advance();
      }
    }
    // end of work: a descriptor with the done flag, completed by a plain arrive
    if (!claim()) return;
    if (lane == 0) {
      StageDesc dsc{};
      dsc.bits = kDescDone << 9;
      desc[slot] = dsc;
      mbar_arrive(&full[slot]);
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
  uint32_t ephase = 0;    // phase of the epilogue barrier
  // Meeting point of the pipeline's compute warps (split-K epilogue).  An mbarrier with a bounded
  // wait rather than a named barrier, so that warps that gave up on a timed-out wait cannot
  // leave the others blocked.
  auto epi_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_bar);
    const bool ok = mbar_wait_ring(epi_bar, ephase);
    ephase ^= 1u;
    if (!ok && lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
    return ok;
  };
  float acc[NB][4];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;
  while (true) {
    const int slot = cslot;
    const uint32_t phase = cphase;
    if (++cslot == S) { cslot = 0; cphase ^= 1u; }
    // (a producer that gave up leaves its stage incomplete: this bounded wait then ends the warp)
    if (!mbar_wait_ring(&full[slot], phase)) {
      if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
      return;
    }
    const int4 d0 = *reinterpret_cast<const int4*>(desc + slot);   // first half of the descriptor
    StageDesc dsc;
    dsc.r0 = d0.x; dsc.g = d0.y; dsc.nt = d0.z; dsc.bits = d0.w;
    const int dflags = desc_flags(dsc);
    if (dflags & kDescDone) return;
    const int g = dsc.g;
    const int gc = desc_gc(dsc);
    const int mt = desc_mt(dsc);
    const uint8_t* xs = smem + L.x_off + slot * L.x_bytes;
    const uint8_t* qs = smem + L.q_off + slot * L.q_bytes;
    const uint8_t* ss = smem + L.sc_off + slot * L.sc_bytes;
    // scales of rows rlo / rhi for the stage's 8 groups, two bf16 per word
    uint32_t slo[4], shi[4];
    if (SCALE == kScaleTma) {
      const uint4 vlo = *reinterpret_cast<const uint4*>(ss + rlo * 16);
      const uint4 vhi = *reinterpret_cast<const uint4*>(ss + rhi * 16);
      slo[0] = vlo.x; slo[1] = vlo.y; slo[2] = vlo.z; slo[3] = vlo.w;
      shi[0] = vhi.x; shi[1] = vhi.y; shi[2] = vhi.z; shi[3] = vhi.w;
    } else if (SCALE == kScaleBlock) {
      // block rows hold all kg groups (kg even, g a multiple of 8: 4-byte aligned pairs)
      const uint32_t* plo = reinterpret_cast<const uint32_t*>(ss + (rlo * A.kg + g) * 2);
      const uint32_t* phi = reinterpret_cast<const uint32_t*>(ss + (rhi * A.kg + g) * 2);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        slo[p] = 2 * p < gc ? plo[p] : 0u;
        shi[p] = 2 * p < gc ? phi[p] : 0u;
      }
    } else {
      const int dnt = dsc.nt, de = desc[slot].e;
      const int64_t grow_lo = tile_row_valid(A, dnt, rlo) ? tile_row(A, de, dnt, rlo) : tile_row(A, de, dnt, 0);
      const int64_t grow_hi = tile_row_valid(A, dnt, rhi) ? tile_row(A, de, dnt, rhi) : tile_row(A, de, dnt, 0);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int ga = g + 2 * p, gb = g + 2 * p + 1;
        const uint32_t l0 = 2 * p < gc ? ldg_u16(A.scales + grow_lo * A.kg + ga) : 0;
        const uint32_t l1 = 2 * p + 1 < gc ? ldg_u16(A.scales + grow_lo * A.kg + gb) : 0;
        const uint32_t h0 = 2 * p < gc ? ldg_u16(A.scales + grow_hi * A.kg + ga) : 0;
        const uint32_t h1 = 2 * p + 1 < gc ? ldg_u16(A.scales + grow_hi * A.kg + gb) : 0;
        slo[p] = l0 | (l1 << 16);
        shi[p] = h0 | (h1 << 16);
      }
    }
    // Word (row r, group gi, quad position tq) sits at chunk gi ^ (r % 8) of the 128-byte row
    // (TMA 128-byte swizzle).  Each extracted fp16 pair is two consecutive k, so k-step 0 takes
    // elements 8tq+0..3 (x pairs .x, .y) and k-step 1 elements 8tq+4..7 (.z, .w).
    // Rows rlo and rhi share the swizzle phase (rlo % 8): one address per group.  Shared
    // address of (row rlo, chunk c, word tq) = stage + rlo*128 + ((c ^ r7) << 4) + 4 tq; the
    // stage and row bases have bits 4-6 clear, so this is base ^ (c << 4) with the r7 part
    // folded into base: one XOR per group.
    const uint32_t abase = smem_u32(smem + slot * kCodeBytes) + ((rlo * 128 + 4 * tq) ^ (r7 << 4));
    if (NB == 1) {
      // one token block: extraction fused into the MMAs
      const uint8_t* xrow = xs + gid * kXPitch + tq * 16;
      const uint8_t* qrow = qs + tq * kQPitch;      // row pair (2tq, 2tq + 1)
      const uint32_t e1024 = 0x64006400u;
#pragma unroll
      for (int gi = 0; gi < kGS; ++gi) {
        const uint32_t aw = abase ^ static_cast<uint32_t>(gi << 4);
        const uint32_t wlo = lds32(aw);
        const uint32_t whi = lds32(aw + kDwBytes);
        const uint4 xv = *reinterpret_cast<const uint4*>(xrow + gi * 64);
        const float4 cq = *reinterpret_cast<const float4*>(qrow + gi * 16);
        const float c[4] = {cq.x, cq.y, cq.z, cq.w};
        float d[4];
        mma_nib(d, wlo, whi, xv.x, xv.y, c, e1024);
        mma_nib(d, wlo >> 8, whi >> 8, xv.z, xv.w, d, e1024);
        const uint32_t sl = (gi & 1) ? (slo[gi >> 1] & 0xFFFF0000u) : (slo[gi >> 1] << 16);
        const uint32_t sh = (gi & 1) ? (shi[gi >> 1] & 0xFFFF0000u) : (shi[gi >> 1] << 16);
        acc[0][0] = fmaf(__uint_as_float(sl), d[0], acc[0][0]);
        acc[0][1] = fmaf(__uint_as_float(sl), d[1], acc[0][1]);
        acc[0][2] = fmaf(__uint_as_float(sh), d[2], acc[0][2]);
        acc[0][3] = fmaf(__uint_as_float(sh), d[3], acc[0][3]);
      }
    } else {
      // Passes of kGP groups: extract rows rlo / rhi into MMA A fragments once, then run the
      // token blocks.
      const int nblk = (mt + 7) >> 3;
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
          const uint32_t wlo8 = wlo >> 8, whi8 = whi >> 8;
          fa[i][0] = nib_f16x2_lo(wlo);      // k-step 0: elements (0,1) | (2,3) x 16
          fa[i][1] = nib_f16x2_lo(whi);
          fa[i][2] = nib_f16x2_hi(wlo);
          fa[i][3] = nib_f16x2_hi(whi);
          fa[i][4] = nib_f16x2_lo(wlo8);     // k-step 1: elements (4,5) | (6,7) x 16
          fa[i][5] = nib_f16x2_lo(whi8);
          fa[i][6] = nib_f16x2_hi(wlo8);
          fa[i][7] = nib_f16x2_hi(whi8);
          const uint32_t sl = (gi & 1) ? (slo[gi >> 1] & 0xFFFF0000u) : (slo[gi >> 1] << 16);
          const uint32_t sh = (gi & 1) ? (shi[gi >> 1] & 0xFFFF0000u) : (shi[gi >> 1] << 16);
          fsl[i] = __uint_as_float(sl);
          fsh[i] = __uint_as_float(sh);
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < nblk) {
            const uint8_t* xrow = xs + (b * 8 + gid) * kXPitch + tq * 16;
            const uint8_t* qrow = qs + (b * 4 + tq) * kQPitch;    // row pair (b*8 + 2tq, +1)
#pragma unroll
            for (int i = 0; i < kGP; ++i) {
              const uint4 xv = *reinterpret_cast<const uint4*>(xrow + (h + i) * 64);
              const float4 cq = *reinterpret_cast<const float4*>(qrow + (h + i) * 16);
              const uint32_t a0[4] = {fa[i][0], fa[i][1], fa[i][2], fa[i][3]};
              const uint32_t a1[4] = {fa[i][4], fa[i][5], fa[i][6], fa[i][7]};
              const float c[4] = {cq.x, cq.y, cq.z, cq.w};
              float d[4];
              mma_f16_16816(d, a0, xv.x, xv.y, c);
              mma_f16_16816(d, a1, xv.z, xv.w, d);
              acc[b][0] = fmaf(fsl[i], d[0], acc[b][0]);
              acc[b][1] = fmaf(fsl[i], d[1], acc[b][1]);
              acc[b][2] = fmaf(fsh[i], d[2], acc[b][2]);
              acc[b][3] = fmaf(fsh[i], d[3], acc[b][3]);
            }
          }
        }
      }
    }
    const bool last = dflags & kDescLast;
    int sp_last = 0, tile_last = 0;     // the unit's K split and tile id (split-K epilogue)
    if (last) {
      if (A.splits > 1) {
        const int4 d1 = reinterpret_cast<const int4*>(desc + slot)[1];   // before the slot is freed
        sp_last = d1.y;
        tile_last = d1.z;
      }
      // undo the activation rows' power-of-two exponents (token columns 2tq, 2tq + 1 of each
      // block; the multipliers travel with the rows, so no global load waits behind the stream)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int t0 = b * 8 + 2 * tq;
        const float m0 = t0 < mt ? *reinterpret_cast<const float*>(xs + t0 * kXPitch + kXBlock) : 0.f;
        const float m1 = t0 + 1 < mt ? *reinterpret_cast<const float*>(xs + (t0 + 1) * kXPitch + kXBlock) : 0.f;
        acc[b][0] *= m0; acc[b][2] *= m0;
        acc[b][1] *= m1; acc[b][3] *= m1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (!last) continue;

    // --------------------------- epilogue (last stage of a unit) ---------------------------
    const int64_t r0 = dsc.r0;
    const int nt = dsc.nt;
    if (A.splits == 1) {
      // straight from registers: thread holds rows rlo / rhi for tokens 2tq, 2tq + 1 of each block
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int t0 = b * 8 + 2 * tq;
        if (gelu) {
          const int Nh = A.N >> 1;
          const int j = nt * kHalf + warp * 8 + gid;
          if (j < Nh) {
            if (t0 < mt)
              A.out[(r0 + t0) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][0]) * acc[b][2]);
            if (t0 + 1 < mt)
              A.out[(r0 + t0 + 1) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][1]) * acc[b][3]);
          }
        } else {
          const int nlo = nt * kBN + rlo, nhi = nlo + 8;
          if (t0 < mt) {
            if (nlo < A.N) A.out[(r0 + t0) * A.N + nlo] = f32_to_bf16_bits(acc[b][0]);
            if (nhi < A.N) A.out[(r0 + t0) * A.N + nhi] = f32_to_bf16_bits(acc[b][2]);
          }
          if (t0 + 1 < mt) {
            if (nlo < A.N) A.out[(r0 + t0 + 1) * A.N + nlo] = f32_to_bf16_bits(acc[b][1]);
            if (nhi < A.N) A.out[(r0 + t0 + 1) * A.N + nhi] = f32_to_bf16_bits(acc[b][3]);
          }
        }
      }
    } else {
      // split-K: float32 partials through shared memory, then the last pipeline to finish its
      // part of the tile reduces them in split order (and applies the GELU gate)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int t0 = b * 8 + 2 * tq;
        ep[t0 * kEpPitch + rlo] = acc[b][0];
        ep[(t0 + 1) * kEpPitch + rlo] = acc[b][1];
        ep[t0 * kEpPitch + rhi] = acc[b][2];
        ep[(t0 + 1) * kEpPitch + rhi] = acc[b][3];
      }
      if (!epi_sync()) return;
      const int ctid = warp * 32 + lane;
      const int Nh = A.N >> 1;
      // partial column of tile row c (GELU: rows 0..63 gate j, 64..127 up j of outputs j)
      auto pcol = [&](int c, bool& ok) -> int {
        if (gelu) {
          const int j = nt * kHalf + (c & (kHalf - 1));
          ok = j < Nh;
          return c < kHalf ? j : Nh + j;
        }
        const int n = nt * kBN + c;
        ok = n < A.N;
        return n;
      };
      if (!flags[0]) {
        for (int idx = ctid; idx < mt * kBN; idx += kWarps * 32) {
          const int t = idx / kBN, c = idx % kBN;
          bool ok;
          const int n = pcol(c, ok);
          if (ok)
            A.partial[(static_cast<int64_t>(sp_last) * A.rows + r0 + t) * A.N + n] = ep[t * kEpPitch + c];
        }
      }
      __threadfence();
      if (!epi_sync()) return;
      if (ctid == 0) {
        int last = 0;
        if (!flags[0]) {
          const int prev = atomicAdd(&A.counters[tile_last], 1);
          last = (prev == A.splits - 1);
          if (last) A.counters[tile_last] = 0;
        }
        flags[1] = last;
      }
      if (!epi_sync()) return;
      if (flags[1]) {
        __threadfence();
        const int64_t ps = A.rows * A.N;
        // the partials of up to 8 splits are loaded together, then summed in split order
        auto sum_col = [&](int t, int n) -> float {
          const float* pp = A.partial + (r0 + t) * A.N + n;
          float sum = 0.f;
          for (int sp0 = 0; sp0 < A.splits; sp0 += 8) {
            float pv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) pv[q] = sp0 + q < A.splits ? __ldcg(pp + (sp0 + q) * ps) : 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) sum += pv[q];
          }
          return sum;
        };
        if (gelu) {
          for (int idx = ctid; idx < mt * kHalf; idx += kWarps * 32) {
            const int t = idx / kHalf, c = idx % kHalf;
            const int j = nt * kHalf + c;
            if (j < Nh)
              A.out[(r0 + t) * Nh + j] = f32_to_bf16_bits(gelu_tanh(sum_col(t, j)) * sum_col(t, Nh + j));
          }
        } else {
          const int n0 = nt * kBN;
          for (int idx = ctid; idx < mt * kBN; idx += kWarps * 32) {
            const int t = idx / kBN, c = idx % kBN;
            if (n0 + c < A.N) A.out[(r0 + t) * A.N + n0 + c] = f32_to_bf16_bits(sum_col(t, n0 + c));
          }
        }
      }
      if (!epi_sync()) return;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = 0.f;
  }
}

// Preparation pass: one warp per routed row r (row r of `a`, or row a_row_of_pair[r] / k_div,
// checked).  Pass 1 finds the row's largest finite |x| and its exponent f (largest in
// [2^14, 2^15)); pass 2 writes, per 256-k block j, lane l's 8 elements 8l..8l+7 as fp16
// (elements 2, 3, 6, 7 with 2^(f-4), the rest with 2^f) and the correction of group l / 4:
// c = -(1032 * (x'0 + x'1 + x'4 + x'5) + 1152 * (x'2 + x'3 + x'6 + x'7)) summed over its 4 lanes
// (from the stored fp16 values), into the quad slots 0, 2 of row r and 1, 3 of row r - 1.
// Elements past K are written as zero.  Every block also carries the row's multiplier 2^-f
// (bytes 512..515), so that a unit's epilogue finds it next to its last stage.
__global__ void __launch_bounds__(256)
stream_prep_kernel(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair, int k_div,
                   int64_t a_rows, int64_t rows, int K, uint8_t* __restrict__ xw, int64_t stride,
                   int32_t* __restrict__ counters, int n_counters, int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = K >> 3;                          // 8-element chunks in the row
  const int nblk = (K + kGS * 32 - 1) / (kGS * 32);
  pdl_trigger();
  pdl_wait();
  // the GEMM's split-K arrival counters start at zero whatever the workspace held before
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_counters; i += gridDim.x * blockDim.x)
    counters[i] = 0;
  for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    int64_t src = r;
    if (a_row_of_pair) {
      src = __ldg(a_row_of_pair + r) / k_div;
      if (src < 0 || src >= a_rows) {
        if (lane == 0) set_status(dev_status, W4_ERR_INVALID_ARG);
        src = 0;
      }
    }
    const uint4* row = reinterpret_cast<const uint4*>(a + src * K);
    // Lane l holds chunk l of up to kPB 256-k blocks at a time, all loads of a batch in flight
    // together; a row of at most kPB blocks is read once.
    uint4 v[kPB];
    uint32_t m = 0;
    for (int j0 = 0; j0 < nblk; j0 += kPB) {
#pragma unroll
      for (int t = 0; t < kPB; ++t) {
        const int i = (j0 + t) * 32 + lane;
        v[t] = i < nv ? __ldg(row + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int t = 0; t < kPB; ++t) {
        const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = w[q] & 0x7FFFu, hi = (w[q] >> 16) & 0x7FFFu;
          if (lo < 0x7F80u) m = max(m, lo);
          if (hi < 0x7F80u) m = max(m, hi);
        }
      }
    }
    m = __reduce_max_sync(0xffffffffu, m);
    const int f = shift_for(m, 14);
    const float m1 = pow2f(f), m16 = pow2f(f - 4);
    uint8_t* dst = xw + r * stride;
    for (int j0 = 0; j0 < nblk; j0 += kPB) {
      if (nblk > kPB) {                          // long rows: the batch again (from L1 / L2)
#pragma unroll
        for (int t = 0; t < kPB; ++t) {
          const int i = (j0 + t) * 32 + lane;
          v[t] = i < nv ? __ldg(row + i) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int t = 0; t < kPB; ++t) {
        const int j = j0 + t;
        if (j >= nblk) break;
        const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
        uint32_t h[4];
        f16_pairs_l1(w, m1, m16, h);             // (x0, x4), (x1, x5)/16, (x2, x6), (x3, x7)/16
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h[0]));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h[1]));
        const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&h[2]));
        const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&h[3]));
        float part = 1032.f * ((f0.x + f0.y) + (f2.x + f2.y)) + 1152.f * ((f1.x + f1.y) + (f3.x + f3.y));
        const uint4 o = make_uint4(h[0], h[1], h[2], h[3]);
        uint8_t* blk = dst + static_cast<int64_t>(j) * kPrepStage;
        *reinterpret_cast<uint4*>(blk + lane * 16) = o;
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if ((lane & 3) == 0) {
          const float c = -part;
          float* q = reinterpret_cast<float*>(blk + kXCopy + (lane >> 2) * 16);
          q[0] = c;
          q[2] = c;
          if (r + 1 == rows) { q[1] = 0.f; q[3] = 0.f; }
          if (r > 0) {
            float* qp = reinterpret_cast<float*>(blk - stride + kXCopy + (lane >> 2) * 16);
            qp[1] = c;
            qp[3] = c;
          }
        }
      }
    }
    for (int j = lane; j < nblk; j += 32)
      *reinterpret_cast<float4*>(dst + static_cast<int64_t>(j) * kPrepStage + kXBlock) =
          make_float4(pow2f(-f), 0.f, 0.f, 0.f);
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

// Ring depth and offsets for one launch: each of the CTA's two pipelines gets half of the shared
// memory left next to the unit table, with as many stages (up to kMaxStages) as fit.
static w4::Layout make_layout(int MT, int scale_mode, int kg, int E, bool split) {
  // every per-stage region is a multiple of 128 bytes, so each region's base keeps the 128-byte
  // alignment a TMA tile destination needs whatever the ring depth
  w4::Layout L{};
  L.x_bytes = (MT * w4::kXPitch + 127) & ~127;
  L.q_bytes = ((MT / 2) * w4::kQPitch + 127) & ~127;
  L.sc_bytes = scale_mode == w4::kScaleTma ? 2 * w4::kHalf * w4::kGS * 2
             : scale_mode == w4::kScaleBlock ? 2 * w4::kHalf * kg * 2 : 16;
  L.sc_bytes = (L.sc_bytes + 127) & ~127;
  const int table_bytes = (E + 1) * 8;
  const int ep_bytes = split ? MT * w4::kEpPitch * 4 : 0;
  const int budget = ((w4::kSmemPerCta - 1024 - table_bytes) / w4::kPipes) & ~1023;   // per pipeline
  const int fixed = ep_bytes + w4::kMaxStages * w4::kDescBytes + (2 * w4::kMaxStages + 1) * 8 + 16 + 128;
  const int per_stage = w4::kCodeBytes + L.x_bytes + L.q_bytes + L.sc_bytes;
  int S = (budget - fixed) / per_stage;
  if (S > w4::kMaxStages) S = w4::kMaxStages;
  L.stages = S;
  L.x_off = S * w4::kCodeBytes;
  L.q_off = L.x_off + S * L.x_bytes;
  L.sc_off = L.q_off + S * L.q_bytes;
  int off = L.sc_off + S * L.sc_bytes;
  L.desc_off = off;
  off += S * w4::kDescBytes;
  L.ep_off = split ? off : -1;
  off += ep_bytes;
  L.bar_off = (off + 7) & ~7;
  off = L.bar_off + (2 * S + 1) * 8;
  L.flag_off = off;
  off += 16;
  L.pipe_bytes = (off + 1023) & ~1023;
  L.table_off = w4::kPipes * L.pipe_bytes;
  L.total = L.table_off + table_bytes + 1024;    // + alignment slack of the dynamic base
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
  // Split K into as many parts as keep all units within one wave of the pipelines (long units
  // stream better than many short ones: a K = 4096 GEMV measured fastest with two splits, and a
  // second wave of split units costs more than it saves), with at least two stages per part and
  // float32 partials below ~1/8 of the weight bytes.  Grouped calls count the token blocks the
  // most spread-out routing can produce: at most one per row, and at most one per expert plus
  // one per MT rows.
  const int64_t ntb = dense ? (rows + p.MT - 1) / p.MT
                            : std::min<int64_t>(rows, static_cast<int64_t>(E) + rows / p.MT);
  const int64_t units = std::max<int64_t>(1, ntb * p.n_tiles);
  const double wbytes = static_cast<double>(E) * N * K * 0.5625;
  int64_t sp = static_cast<int64_t>(w4::kPipes) * sm_count / units;
  sp = std::min<int64_t>(sp, kstages / 2);
  while (sp > 1 && static_cast<double>(sp) * rows * N * 4.0 > wbytes / 8.0) --sp;
  p.splits = sp > 1 ? static_cast<int>(sp) : 1;
  p.stages_per_split = (kstages + p.splits - 1) / p.splits;
  p.splits = (kstages + p.stages_per_split - 1) / p.stages_per_split;
  return p;
}

// Workspace: the prepared activation rows [rows][K/256 blocks][656 bytes] (256-byte aligned);
// with split-K then the per-tile arrival counters (cleared by every launch) and the float32
// partials [splits, rows, N].
static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

static int64_t prep_stride(int K) {
  return static_cast<int64_t>((K + w4::kGS * 32 - 1) / (w4::kGS * 32)) * w4::kPrepStage;
}

static size_t prep_bytes(int64_t rows, int K) {
  return align256(static_cast<size_t>(rows) * prep_stride(K));
}

// one arrival counter per (expert, token block, weight tile): at most min(E, rows) + rows / MT
// token blocks over all experts
static size_t counters_bytes(const StreamPlan& p, int64_t rows, int E) {
  const int64_t ntb = std::min<int64_t>(E, rows) + (rows + p.MT - 1) / p.MT;
  return align256(static_cast<size_t>(ntb * p.n_tiles) * sizeof(int32_t));
}

size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  if (rows <= 0) return 0;
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  size_t b = prep_bytes(rows, K);
  if (p.splits > 1) b += counters_bytes(p, rows, E) + static_cast<size_t>(p.splits) * rows * N * sizeof(float);
  return b;
}

template <int MT, bool GELU, int SCALE>
static w4_status launch_one(const CUtensorMap& tmap, const CUtensorMap& smap, const w4::StreamArgs& A,
                            int sm_count, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel<MT, GELU, SCALE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, w4::kSmemPerCta) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  return launch_pdl(w4::stream_gemm_kernel<MT, GELU, SCALE>, dim3(sm_count), dim3(w4::kThreads),
                    A.L.total, stream, tmap, smap, A) == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

template <int MT, bool GELU>
static w4_status launch_scale(int scale_mode, const CUtensorMap& tmap, const CUtensorMap& smap,
                              const w4::StreamArgs& A, int sm_count, cudaStream_t stream) {
  if (scale_mode == w4::kScaleTma) return launch_one<MT, GELU, w4::kScaleTma>(tmap, smap, A, sm_count, stream);
  if (scale_mode == w4::kScaleBlock) return launch_one<MT, GELU, w4::kScaleBlock>(tmap, smap, A, sm_count, stream);
  return launch_one<MT, GELU, w4::kScaleLdg>(tmap, smap, A, sm_count, stream);
}

w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count) {
  const bool dense = (offsets == nullptr);
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  w4::StreamArgs A{};
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32; A.rows = rows; A.epi = epi; A.out = out;
  A.splits = p.splits; A.stages_per_split = p.stages_per_split; A.n_tiles = p.n_tiles;
  A.dev_status = dev_status;
  {
    // grouped calls whose experts' weights fit in half of L2 (a few decode tokens): prefetch
    // every stage at the start (measured: one-token 30-layer decode 1.17 -> 1.11 ms per step; a
    // dense K = 4096 GEMV got slower, its ring's first loads queue behind the prefetches)
    const double touched = static_cast<double>(std::min<int64_t>(E, rows)) * N * K * 0.5625;
    A.pf_all = !dense && touched <= 64.0 * (1 << 20);
  }
  // Scale staging: 2-D TMA when a scale row is a whole number of 16-byte chunks; else the tile's
  // contiguous 64-row scale blocks by bulk copy when they are 16-byte aligned and small; else
  // direct loads.
  const bool s16 = (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
  int scale_mode;
  if (A.kg % 8 == 0 && s16) {
    scale_mode = w4::kScaleTma;
  } else if (A.kg % 2 == 0 && A.kg <= w4::kBlockMaxKg && N % 8 == 0 && s16 &&
             (epi == W4_EPI_GELU_GATE ? (N / 2) % w4::kHalf == 0 : N % w4::kBN == 0)) {
    // (whole tiles only: the 64-row blocks are plain bulk copies and must stay inside the array)
    scale_mode = w4::kScaleBlock;
  } else {
    scale_mode = w4::kScaleLdg;
  }
  A.L = make_layout(p.MT, scale_mode, A.kg, E, p.splits > 1);
  if (A.L.stages < 2) return W4_ERR_UNSUPPORTED;
  if (rows == 0) return W4_OK;
  const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count);
  if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  A.xw = wsb;
  A.xw_stride = prep_stride(K);
  if (p.splits > 1) {
    uint8_t* cbase = wsb + prep_bytes(rows, K);
    const size_t cb = counters_bytes(p, rows, E);
    A.counters = reinterpret_cast<int32_t*>(cbase);
    A.partial = reinterpret_cast<float*>(cbase + cb);
    // (the preparation pass clears the arrival counters)
  }
  {
    const int kd = k_div > 0 ? k_div : 1;
    const int64_t a_rows = a_row_of_pair ? rows / kd : rows;
    const int64_t blocks = (rows + 7) / 8;
    const int grid = static_cast<int>(blocks < 16LL * sm_count ? blocks : 16LL * sm_count);
    const int n_counters = p.splits > 1 ? static_cast<int>(counters_bytes(p, rows, E) / sizeof(int32_t)) : 0;
    if (launch_pdl(w4::stream_prep_kernel, dim3(grid), dim3(256), 0, stream, a, a_row_of_pair, kd, a_rows,
                   rows, K, wsb, A.xw_stride, A.counters, n_counters, dev_status) != cudaSuccess)
      return W4_ERR_CUDA;
  }
  CUtensorMap tmap, smap;
  std::memset(&smap, 0, sizeof(smap));
  if (!encode_codes_map(&tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  if (scale_mode == w4::kScaleTma &&
      !encode_scales_map(&smap, scales, static_cast<int64_t>(E) * N, A.kg))
    return W4_ERR_CUDA;
  const bool gelu = A.epi == W4_EPI_GELU_GATE;
  if (p.MT == 8)
    return gelu ? launch_scale<8, true>(scale_mode, tmap, smap, A, sm_count, stream)
                : launch_scale<8, false>(scale_mode, tmap, smap, A, sm_count, stream);
  return gelu ? launch_scale<16, true>(scale_mode, tmap, smap, A, sm_count, stream)
              : launch_scale<16, false>(scale_mode, tmap, smap, A, sm_count, stream);
}
