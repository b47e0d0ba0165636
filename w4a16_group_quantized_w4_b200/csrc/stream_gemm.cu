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
//   * Token blocks: the routed rows of each expert (all rows for a dense linear) are cut into
//     blocks of MT (8 or 16) consecutive rows.  A preparation pass (one warp per routed row)
//     writes, for every block and every stage of GS groups (GS * 32 k), one contiguous record:
//     the block's rows as fp16 x' = x * 2^f (f per row, putting its largest |x| in
//     [2^14, 2^15)), the per-group bias corrections of every row pair as quads, and the rows'
//     multipliers 2^-f.  Within every 8 consecutive k the values are stored in the order
//     0, 4, 1, 5, 2, 6, 3, 7 (the order in which a layout-L1 code word is split, see below), the
//     second and fourth pair divided by 16.  A stage's activations then arrive with one bulk copy.
//   * Work unit = (expert e, token block, tile of 128 weight rows, K split).  A persistent grid
//     (one CTA per SM, two independent pipelines of 8 compute warps + 1 producer warp) walks the
//     units; the unit table is a prefix sum over the experts built on the device from
//     expert_offsets (no host synchronisation).
//   * The producer keeps a ring of shared-memory slots full.  One slot = one stage: the 128-row
//     code tile for GS groups (2-D TMA boxes of 64 rows x 128 bytes, 128-byte swizzle), the
//     matching bf16 scales, the block's prepared record and a 32-byte stage descriptor, all
//     completing on the slot's mbarrier.  GS = 16 (512 k) for 8-row blocks, 8 for 16-row blocks:
//     long stages halve the per-stage work of the compute warps (barrier wait, descriptor, scale
//     loads, release) per weight.
//   * A compute warp owns 16 weight rows.  A thread's 32-bit code word (8 nibbles, layout L1)
//     gives four fp16 pairs with one shift and four lop3: nibbles (j, j + 4) become 1024 + u for
//     j = 0, 2 and 1024 + 16 u for j = 1, 3 (exact), against activations stored divided by 16 at
//     those positions, so every product is (bias + u) * x' with bias 1024 or 64 (in units of x').
//     The group's correction quad is the C operand of its first MMA, which removes the bias and
//     the -8 of q = u - 8: d = sum over the group of q * x'.  The group's scale is folded in
//     with one fp32 FMA per accumulator: acc += s_g * d.  The epilogue multiplies by the token's
//     2^-f, read from the unit's last stage.
//   * Epilogue from registers: with the GELU gate each warp's two A-fragment row sets are 8 gate
//     rows and the 8 up rows of the same outputs, so h = gelu(g) * u is formed in the thread that
//     holds both.  When the units would not cover the pipelines (dense GEMVs, grouped calls with
//     a few routed rows), K is split: float32 partials that the last pipeline of the tile
//     reduces in a fixed order (deterministic), applying the GELU gate after the sum.
// Rounding: the products are exact; each MMA sums 16 products of up to (1024 + 240) * 2^15 in
// float32 next to the bias, which the correction cancels, so a group's sum carries an absolute
// error of a few float32 units of its bias term (about 2^-13 of the group's mean |x'| times the
// group size), far inside the bf16 rounding of the output.
#include <cudaTypedefs.h>

#include <cstring>

#include <cuda_fp16.h>

#include "common.cuh"

namespace w4 {

constexpr int kMaxStages = 6;
constexpr int kWarps = 8;                     // compute warps per pipeline
constexpr int kPipes = 2;                     // pipelines per CTA (one CTA per SM)
constexpr int kPipeWarps = kWarps + 1;        // + one producer warp
constexpr int kThreads = kPipes * kPipeWarps * 32;
constexpr int kBN = 16 * kWarps;              // weight rows per tile
constexpr int kHalf = kBN / 2;                // rows per TMA box
constexpr int kBoxG = 8;                      // groups per code box (128 bytes of a row)
constexpr int kBoxBytes = kHalf * 128;        // one 64-row code box
constexpr int kBlockMaxKg = 24;               // scale-block mode: two 64-row blocks of <= 24 groups
constexpr int kEpPitch = kBN + 4;             // floats per token row in the epilogue buffer
constexpr int kPB = 12;                       // preparation pass: 256-k blocks per register batch
// dynamic shared memory of the CTA (227 KB opt-in limit per block)
constexpr int kSmemPerCta = 232448;

enum ScaleMode { kScaleLdg = 0, kScaleBlock = 1, kScaleTma = 2 };

// Prepared record of one token block (MT rows) and one stage (GS groups):
//   [MT rows x rec_xp bytes of x' (GS * 64 bytes, padded so that consecutive rows sit 64 bytes
//    apart in the shared-memory banks)]
//   [quads: group-major, GS x MT/2 row pairs x 16 bytes {c(r), c(r+1), c(r), c(r+1)}]
//   [MT row multipliers 2^-f (float)], padded to 16 bytes
//   [zero-point variant only: group-major, GS x MT/2 row pairs x 8 bytes {Sx(r), Sx(r+1)}, the
//    sum over the group of the row's x' values], padded to 16 bytes.
__host__ __device__ constexpr int rec_xp(int GS) { return GS * 64 + 64; }
__host__ __device__ constexpr int rec_qoff(int MT, int GS) { return MT * rec_xp(GS); }
__host__ __device__ constexpr int rec_moff(int MT, int GS) { return rec_qoff(MT, GS) + GS * (MT / 2) * 16; }
__host__ __device__ constexpr int rec_soff(int MT, int GS) { return (rec_moff(MT, GS) + MT * 4 + 15) & ~15; }
__host__ __device__ constexpr int rec_bytes(int MT, int GS, bool ZP = false) {
  return ZP ? (rec_soff(MT, GS) + GS * (MT / 2) * 8 + 15) & ~15 : rec_soff(MT, GS);
}

// Shared-memory slot of one stage (offsets from the slot base, a multiple of 1024 bytes):
//   codes: GS/8 column boxes x 2 row halves x 8 KB; then the prepared record; then the stage
//   descriptor; then the scales.
__host__ __device__ constexpr int slot_code_bytes(int GS) { return (GS / kBoxG) * 2 * kBoxBytes; }
__host__ __device__ constexpr int slot_act_off(int GS) { return slot_code_bytes(GS); }
__host__ __device__ constexpr int slot_desc_off(int MT, int GS, bool ZP = false) {
  return slot_act_off(GS) + ((rec_bytes(MT, GS, ZP) + 127) & ~127);
}
__host__ __device__ constexpr int slot_sc_off(int MT, int GS, bool ZP = false) { return slot_desc_off(MT, GS, ZP) + 128; }

// Shared-memory layout of one launch (offsets from the 1024-byte aligned base): pipeline p's
// ring at p * pipe_bytes, its split-K epilogue buffer, barriers and flags after the ring; then the
// unit table.
struct Layout {
  int stages;
  int slot_bytes;            // one slot (multiple of 1024)
  int sc_bytes;              // scale bytes per slot
  int ep_off;                // split-K epilogue buffer (MT x kEpPitch floats), or -1
  int red_off;               // k-part hand-over: 2 x (4 m-blocks x MT/8 x 2 tiles x 32 lanes) float4
  int bar_off;               // 2 * stages mbarriers, then the epilogue barrier
  int flag_off;              // 16 bytes
  int pipe_bytes;            // one pipeline's region (multiple of 1024)
  int table_off;             // int table[E + 1], offs[E + 1], blk[E + 1] (shared)
  int total;
};

struct StreamArgs {
  const uint8_t* xw;        // prepared records: [token block][stage][rec_bytes]
  int n_stages;             // stages per row (ceil(K / (GS * 32)))
  const uint16_t* scales;   // [E*N, kgs]: one bf16 per group of 32 << gshift
  const uint8_t* zeros;     // [E*N, kgs] zero-points 0..15 (zero-point variant) or null
  int gshift, kgs;          // scale group = 32 << gshift elements; scales per row
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
  uint64_t wait_ns;         // limit of every bounded wait
  int stall_after;          // fault injection for tests: producers stop after this many stages (< 0: never)
};

struct Unit {
  int e, tb, nt, sp;
  int64_t r0;
  int mt;
  int j0, j1;             // stages [j0, j1) of the unit
  int tile;               // dense id of (e, tb, nt)
  int blk;                // token block id (prepared-record index)
};

// Stage descriptor written by the producer into the slot, read by the compute warps after the
// slot's full barrier: {r0, first group, weight tile, mt | groups << 5 | flags << 10} in the first
// 16 bytes (read every stage), {expert, K split, tile id, 0} in the second (read only by the
// split-K epilogue and the direct-load scale mode).  The tile id numbers the (expert, token
// block, weight tile) triples 0.. densely; the split-K arrival counters are indexed by it.
enum : int { kDescFirst = 1, kDescLast = 2, kDescDone = 4 };
struct __align__(16) StageDesc {
  int r0;
  int g;
  int nt;
  int bits;
  int e, sp, tile, pad;
};
__device__ __forceinline__ int desc_mt(int bits) { return bits & 31; }
__device__ __forceinline__ int desc_gc(int bits) { return (bits >> 5) & 31; }
__device__ __forceinline__ int desc_flags(int bits) { return (bits >> 10) & 7; }

// Unit u -> (expert, token block, tile, split); `table`, `offs`, `blk` live in shared memory.
template <int MT>
__device__ __forceinline__ void decode_unit(const StreamArgs& A, const int* table, const int* offs,
                                            const int* blk, int64_t u, Unit& U) {
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
  U.blk = blk[U.e] + U.tb;
  U.j0 = U.sp * A.stages_per_split;
  U.j1 = min(A.n_stages, U.j0 + A.stages_per_split);
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
// nibbles (0, 4) / (2, 6) as 1024 + u, nibbles (1, 5) / (3, 7) as 1024 + 16 u (exact) -- times
// the activation pairs (b0, b1), plus c.  The extraction sits in the same asm block as the MMA so
// the fragment registers live only across it.  The exponent pattern 0x64006400 comes in as a
// register (one immediate per lop3).
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

// bf16 scale of group gi from the packed pairs w[] (group 2p in the low half of w[p])
__device__ __forceinline__ float scale_of(const uint32_t* w, int gi) {
  return __uint_as_float((gi & 1) ? (w[gi >> 1] & 0xFFFF0000u) : (w[gi >> 1] << 16));
}

template <int MT, int GS, bool GELU, int SCALE, bool ZP>
__global__ void __launch_bounds__(kThreads, 1)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, StreamArgs A) {
  constexpr int kActOff = slot_act_off(GS);
  constexpr int kDescOff = slot_desc_off(MT, GS, ZP);
  constexpr int kScOff = slot_sc_off(MT, GS, ZP);
  constexpr int kRec = rec_bytes(MT, GS, ZP);
  constexpr int kSOff = rec_soff(MT, GS);
  constexpr int kXP = rec_xp(GS);
  constexpr int kQOff = rec_qoff(MT, GS);
  constexpr int kMOff = rec_moff(MT, GS);
  constexpr int NB = MT / 8;                    // token blocks of 8 (the MMA's n)
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
  int* table = reinterpret_cast<int*>(smem0 + L.table_off);
  int* offs = table + (A.E + 1);
  int* blk = offs + (A.E + 1);

  // This kernel's only direct predecessor is its preparation pass, which lets it launch only
  // once everything before the pass (the routing among it) has completed.  So the routing and
  // the weights may be read at once: the producers issue the first lap's weight loads right away
  // and wait for the preparation pass only before its activation copies (below), so the weight
  // stream starts while the pass still runs.  No other thread touches memory the pass writes
  // before it has consumed a stage that its producer issued after waiting.

  // unit table: table[e] = first unit of expert e, table[E] = total; offsets copied to offs[];
  // blk[e] = first token block of expert e.  Offsets that are not non-decreasing from 0 to rows
  // make the launch a no-op (W4_ERR_INVALID_ARG).
  if (warp_all == 0) {
    int run = 0, brun = 0;
    bool bad = false;
    if (A.offsets && lane == 0) bad = (A.offsets[0] != 0) || (A.offsets[A.E] != A.rows);
    for (int base = 0; base < A.E; base += 32) {
      const int e = base + lane;
      int cnt = 0, nb = 0;
      if (e < A.E) {
        const int64_t o0 = A.offsets ? A.offsets[e] : 0;
        const int64_t o1 = A.offsets ? A.offsets[e + 1] : A.rows;
        if (o1 < o0 || o0 < 0 || o1 > A.rows) bad = true;
        const int64_t ntb = o1 > o0 ? (o1 - o0 + MT - 1) / MT : 0;
        nb = static_cast<int>(ntb);
        cnt = static_cast<int>(ntb * A.n_tiles * A.splits);
        offs[e] = static_cast<int>(o0);
        if (e == A.E - 1) offs[A.E] = static_cast<int>(o1);
      }
      int incl = cnt, bincl = nb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        const int bv = __shfl_up_sync(0xffffffffu, bincl, o);
        if (lane >= o) { incl += v; bincl += bv; }
      }
      if (e < A.E) { table[e] = run + incl - cnt; blk[e] = brun + bincl - nb; }
      run += __shfl_sync(0xffffffffu, incl, 31);
      brun += __shfl_sync(0xffffffffu, bincl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) { table[A.E] = bad ? 0 : run; blk[A.E] = brun; }
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
    if (lane != 0) return;
    prefetch_tmap(&tmap_codes);
    if (SCALE == kScaleTma) prefetch_tmap(&tmap_scales);
    int slot = 0;
    uint32_t phase = 0;        // phase of the empty barrier to wait for on the next lap
    bool first_lap = true;
    int64_t issued = 0;        // stages issued so far
    // Before an early exit: wait (bounded) until the copies of the last S stages issued have
    // landed, so that no bulk copy still writes into this CTA's shared memory after it exits.
    // Stage i used slot i % S and completes phase (i / S) of that slot's full barrier.
    auto drain = [&]() {
      for (int64_t i = issued > S ? issued - S : 0; i < issued; ++i)
        mbar_wait_ring(&full[i % S], static_cast<uint32_t>((i / S) & 1), A.wait_ns);
    };
    // claims the next ring slot (false: a wait timed out or the compute warps gave up)
    auto claim = [&]() -> bool {
      if (!first_lap) {
        if (!mbar_wait_ring(&empty[slot], phase, A.wait_ns) || flags[0]) {
          set_status(A.dev_status, W4_ERR_TIMEOUT);
          flags[0] = 1;
          drain();
          return false;
        }
      }
      if (A.stall_after >= 0 && issued >= A.stall_after) {   // (tests: the consumers' waits run out)
        drain();
        return false;
      }
      return true;
    };
    auto advance = [&]() { ++issued; if (++slot == S) { slot = 0; if (!first_lap) phase ^= 1u; first_lap = false; } };
    // the activation copies of the first lap, deferred until the preparation pass writing them
    // has completed
    struct Deferred { uint8_t* dst; const uint8_t* src; uint32_t bytes; uint64_t* bar; };
    Deferred def[2 * kMaxStages];
    int ndef = 0;
    bool waited = false;
    auto act_copy = [&](uint8_t* dst, const uint8_t* src, uint32_t bytes, uint64_t* bar) {
      if (waited) bulk_g2s(dst, src, bytes, bar);
      else def[ndef++] = Deferred{dst, src, bytes, bar};
    };
    auto flush = [&]() {
      if (waited) return;
      pdl_wait();
      waited = true;
      for (int i = 0; i < ndef; ++i) bulk_g2s(def[i].dst, def[i].src, def[i].bytes, def[i].bar);
      ndef = 0;
    };
    if (A.pf_all) {
      // weights that fit in L2 several times over: ask for all of this pipeline's code and scale
      // tiles now, so DRAM streams them at full rate while the ring fills from L2
      for (int64_t u = vb; u < total_units; u += nvb) {
        Unit U;
        decode_unit<MT>(A, table, offs, blk, u, U);
        const int32_t ra = static_cast<int32_t>(tile_row(A, U.e, U.nt, 0));
        const int32_t rb = static_cast<int32_t>(tile_row(A, U.e, U.nt, kHalf));
        for (int j = U.j0; j < U.j1; ++j) {
          for (int s = 0; s < GS / kBoxG; ++s) {
            const int gs = j * GS + s * kBoxG;
            if (gs >= A.kg) break;
            tma_prefetch_2d(&tmap_codes, gs * 4, ra);
            tma_prefetch_2d(&tmap_codes, gs * 4, rb);
          }
          if (SCALE == kScaleTma) {
            tma_prefetch_2d(&tmap_scales, j * GS, ra);
            tma_prefetch_2d(&tmap_scales, j * GS, rb);
          }
        }
        if (SCALE == kScaleBlock) {
          bulk_prefetch_l2(A.scales + static_cast<int64_t>(ra) * A.kg, kHalf * A.kg * 2);
          bulk_prefetch_l2(A.scales + static_cast<int64_t>(rb) * A.kg, kHalf * A.kg * 2);
        }
      }
    }
    const uint32_t sbytes = SCALE == kScaleTma ? 2 * kHalf * GS * 2
                          : SCALE == kScaleBlock ? 2 * kHalf * A.kg * 2 : 0;
    for (int64_t u = vb; u < total_units; u += nvb) {
      Unit U;
      decode_unit<MT>(A, table, offs, blk, u, U);
      const int64_t row_a = tile_row(A, U.e, U.nt, 0);
      const int64_t row_b = tile_row(A, U.e, U.nt, kHalf);
      const uint8_t* rec0 = A.xw + static_cast<int64_t>(U.blk) * A.n_stages * kRec;
      // a full block is one copy; a short block copies its rows and then the quads/multipliers
      const uint32_t xbytes = U.mt == MT ? kRec : U.mt * kXP + (kRec - kQOff);
      for (int j = U.j0; j < U.j1; ++j) {
        if (!first_lap) flush();                // (before the first wait that can run out)
        if (!claim()) return;
        uint8_t* sl = smem + slot * L.slot_bytes;
        const int g = j * GS;
        const int gc = min(GS, A.kg - g);
        const int nbox = (gc + kBoxG - 1) / kBoxG;          // column boxes holding any group
        StageDesc dsc;
        dsc.r0 = static_cast<int>(U.r0);
        dsc.g = g;
        dsc.nt = U.nt;
        const int fl = (j == U.j0 ? kDescFirst : 0) | (j + 1 == U.j1 ? kDescLast : 0);
        dsc.bits = U.mt | (gc << 5) | (fl << 10);
        dsc.e = U.e;
        dsc.sp = U.sp;
        dsc.tile = U.tile;
        dsc.pad = 0;
        *reinterpret_cast<StageDesc*>(sl + kDescOff) = dsc;
        // the arrive releases the descriptor written above
        mbar_arrive_expect_tx(&full[slot], nbox * 2 * kBoxBytes + sbytes + xbytes);
        for (int s = 0; s < nbox; ++s) {
          tma_load_2d(sl + (2 * s) * kBoxBytes, &tmap_codes, (g + s * kBoxG) * 4,
                      static_cast<int32_t>(row_a), &full[slot]);
          tma_load_2d(sl + (2 * s + 1) * kBoxBytes, &tmap_codes, (g + s * kBoxG) * 4,
                      static_cast<int32_t>(row_b), &full[slot]);
        }
        if (SCALE == kScaleTma) {
          tma_load_2d(sl + kScOff, &tmap_scales, g, static_cast<int32_t>(row_a), &full[slot]);
          tma_load_2d(sl + kScOff + kHalf * GS * 2, &tmap_scales, g, static_cast<int32_t>(row_b), &full[slot]);
        } else if (SCALE == kScaleBlock) {
          const uint32_t bb = kHalf * A.kg * 2;
          bulk_g2s(sl + kScOff, A.scales + row_a * A.kg, bb, &full[slot]);
          bulk_g2s(sl + kScOff + bb, A.scales + row_b * A.kg, bb, &full[slot]);
        }
        const uint8_t* rec = rec0 + static_cast<int64_t>(j) * kRec;
        if (U.mt == MT) {
          act_copy(sl + kActOff, rec, kRec, &full[slot]);
        } else {
          act_copy(sl + kActOff, rec, U.mt * kXP, &full[slot]);
          act_copy(sl + kActOff + kQOff, rec + kQOff, kRec - kQOff, &full[slot]);
        }
        advance();
      }
    }
    // end of work: a descriptor with the done flag, completed by a plain arrive
    flush();
    if (!claim()) return;
    StageDesc dsc{};
    dsc.bits = kDescDone << 10;
    *reinterpret_cast<StageDesc*>(smem + slot * L.slot_bytes + kDescOff) = dsc;
    mbar_arrive(&full[slot]);
    return;
  }

  // ------------------------------- compute warps -------------------------------
  // Warp w of the pipeline owns 32 weight rows (two 16-row MMA tiles, m-block w % 4) over one half
  // of every stage's groups (k-part w / 4); the two k-parts of an m-block are summed at the end of
  // each unit (the k-part 1 warp hands its accumulators over through shared memory).  Sharing the
  // activation and correction loads between two MMA tiles halves their shared-memory traffic per
  // weight, and the two tiles' MMA chains are independent.
  // Rows of tile i (i = 0, 1) in this thread's two A-fragment row sets: GELU gate: rlo = gate row
  // 16m + 8i + gid and rhi = the up row of the same output (64 rows further), so the gate is applied
  // in registers; otherwise rlo = 32m + 16i + gid and rhi = rlo + 8.
  const int gid = lane >> 2, tq = lane & 3;
  constexpr bool gelu = GELU;
  const int mb = warp & 3, kp = warp >> 2;
  const int rlo0 = gelu ? 16 * mb + gid : 32 * mb + gid;
  const int r7 = rlo0 & 7;                                  // every row of the thread: same swizzle phase
  constexpr int kDwBytes = GELU ? kBoxBytes : 8 * 128;      // rlo -> rhi
  constexpr int kM1Bytes = GELU ? 8 * 128 : 16 * 128;       // tile 0 -> tile 1
  constexpr int kGW = GS / 2;                               // groups per warp and stage
  // Word (row r, group gi, quad position tq) of a slot: column box gi / 8, row half r / 64, chunk
  // (gi % 8) ^ (r % 8) of the 128-byte row (TMA 128-byte swizzle), word tq.  The slot base and
  // the row part have bits 4-6 clear, so the chunk is one XOR with (gi % 8) << 4 once the row's
  // swizzle phase is folded into the base.
  const uint32_t cbase = static_cast<uint32_t>(((rlo0 >> 6) * kBoxBytes + (rlo0 & 63) * 128 + 4 * tq) ^ (r7 << 4));
  // the thread's four rows: tile i, rlo / rhi
  const int trow[4] = {rlo0, rlo0 + (gelu ? kHalf : 8), rlo0 + (gelu ? 8 : 16), rlo0 + (gelu ? 8 + kHalf : 24)};
  uint32_t soff[4];       // TMA-mode scale offsets of the four rows within a slot
#pragma unroll
  for (int r = 0; r < 4; ++r) soff[r] = kScOff + (trow[r] >> 6) * (kHalf * GS * 2) + (trow[r] & 63) * (GS * 2);
  const uint32_t ring = smem_u32(smem);
  float* ep = reinterpret_cast<float*>(smem + (L.ep_off >= 0 ? L.ep_off : 0));
  float4* red = reinterpret_cast<float4*>(smem + L.red_off);
  int cslot = 0;          // ring slot and mbarrier phase of the current stage
  uint32_t cphase = 0;
  uint32_t ephase = 0;    // phase of the epilogue barrier
  int upar = 0;           // parity of the unit (double-buffered k-part hand-over)
  // Meeting point of the pipeline's compute warps (k-part hand-over, split-K epilogue).  An
  // mbarrier with a bounded wait rather than a named barrier, so that warps that gave up on a
  // timed-out wait cannot leave the others blocked.
  auto epi_sync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_bar);
    const bool ok = mbar_wait_ring(epi_bar, ephase, A.wait_ns);
    ephase ^= 1u;
    if (!ok && lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
    return ok;
  };
  float acc[NB][2][4];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[b][i][q] = 0.f;
  const uint32_t e1024 = 0x64006400u;
  while (true) {
    const int slot = cslot;
    const uint32_t phase = cphase;
    if (++cslot == S) { cslot = 0; cphase ^= 1u; }
    // (a producer that gave up leaves its stage incomplete: this bounded wait then ends the warp)
    if (!mbar_wait_ring(&full[slot], phase, A.wait_ns)) {
      if (lane == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); flags[0] = 1; }
      return;
    }
    const uint32_t sb = ring + slot * L.slot_bytes;
    const uint8_t* sp8 = smem + slot * L.slot_bytes;
    const uint4 d0 = lds128(sb + kDescOff);   // first half of the descriptor
    const int dbits = static_cast<int>(d0.w);
    const int dflags = desc_flags(dbits);
    if (dflags & kDescDone) return;
    const int g = static_cast<int>(d0.y);
    const int gc = desc_gc(dbits);
    const int mt = desc_mt(dbits);
    // A stage's groups are split between the two k-parts: kGW each, or kGW / 2 each when a short
    // last stage loaded only its first column box (GS = 16, at most 8 groups).
    const bool short_stage = GS > kBoxG && gc <= kBoxG;
    const int g0 = short_stage ? kp * (kGW / 2) : kp * kGW;   // this warp's first group
    const int sg0 = short_stage ? 0 : kp * kGW;                // first group of the scales loaded
    {
      // scales of the thread's four rows for its kGW groups, two bf16 per word; zero-points
      // (variant), four bytes per word
      uint32_t sw[4][kGW / 2];
      uint32_t zw[4][ZP ? kGW / 4 : 1];
      if (SCALE == kScaleTma) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t pa = sb + soff[r] + sg0 * 2;
          if (kGW == 8) {
            const uint4 v = lds128(pa);
            sw[r][0] = v.x; sw[r][1 % (kGW / 2)] = v.y; sw[r][2 % (kGW / 2)] = v.z; sw[r][3 % (kGW / 2)] = v.w;
          } else {
            const uint2 v = lds64(pa);
            sw[r][0] = v.x; sw[r][1 % (kGW / 2)] = v.y;
          }
        }
      } else if (SCALE == kScaleBlock) {
        // block rows hold all kg groups (kg even, g + sg0 even: 4-byte aligned pairs)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t* p = reinterpret_cast<const uint32_t*>(
              sp8 + kScOff + (trow[r] >> 6) * (kHalf * A.kg * 2) + ((trow[r] & 63) * A.kg + g + sg0) * 2);
#pragma unroll
          for (int q = 0; q < kGW / 2; ++q) sw[r][q] = sg0 + 2 * q < gc ? p[q] : 0u;
        }
      } else {
        // direct loads (also every other scale group size: group gi of 32 uses scale gi >> gshift)
        const int4 d1 = *reinterpret_cast<const int4*>(sp8 + kDescOff + 16);
        const int dnt = static_cast<int>(d0.z), de = d1.x;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int64_t grow = tile_row_valid(A, dnt, trow[r]) ? tile_row(A, de, dnt, trow[r]) : tile_row(A, de, dnt, 0);
#pragma unroll
          for (int q = 0; q < kGW / 2; ++q) {
            const int ga = g + sg0 + 2 * q;
            const uint32_t l0 = ga - g < gc ? ldg_u16(A.scales + grow * A.kgs + (ga >> A.gshift)) : 0;
            const uint32_t l1 = ga + 1 - g < gc ? ldg_u16(A.scales + grow * A.kgs + ((ga + 1) >> A.gshift)) : 0;
            sw[r][q] = l0 | (l1 << 16);
          }
          if (ZP) {
#pragma unroll
            for (int q = 0; q < kGW / 4; ++q) {
              uint32_t word = 0;
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const int ga = g + sg0 + 4 * q + b;
                const uint32_t zv = ga - g < gc ? __ldg(A.zeros + grow * A.kgs + (ga >> A.gshift)) : 8u;
                word |= zv << (8 * b);
              }
              zw[r][q] = word;
            }
          }
        }
      }
      if (short_stage && kp == 1) {
        // this warp's groups are the second half of the scales loaded
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
          for (int q = 0; q < kGW / 4; ++q) sw[r][q] = sw[r][q + kGW / 4];
          if (ZP) {
#pragma unroll
            for (int q = 0; q < kGW / 8; ++q) zw[r][q] = zw[r][q + kGW / 8];
          }
        }
      }
      // The warp's groups g0 + i, i = 0.. (compile-time): groups 8..15 of a full 16-group stage
      // sit in the second column box; four-group halves (a short stage, or GS = 8) are chunks
      // (4 kp + i) of the first box, i.e. the chunk XOR gains bit 6.  Either way the k-part's
      // offset goes into the stage's base addresses once, and every per-group offset below is an
      // immediate.
      const uint32_t abase = (kGW == 8 && !short_stage) ? sb + cbase + kp * (2 * kBoxBytes)
                                                        : (sb + cbase) ^ static_cast<uint32_t>(kp << 6);
      const uint32_t xg = sb + kActOff + gid * kXP + tq * 16 + g0 * 64;
      const uint32_t qg = sb + kActOff + kQOff + tq * 16 + g0 * (MT / 2) * 16;   // row pair (2tq, 2tq + 1)
      const uint32_t sg = sb + kActOff + kSOff + tq * 8 + g0 * (MT / 2) * 8;      // (zero-point variant)
      const int nblk = NB == 1 ? 1 : (mt + 7) >> 3;
      const int ngw = short_stage ? kGW / 2 : kGW;
#pragma unroll
      for (int i = 0; i < kGW; ++i) {
        if (i >= ngw) break;
        const uint32_t aw = abase ^ static_cast<uint32_t>(i << 4);
        const uint32_t w00 = lds32(aw), w01 = lds32(aw + kDwBytes);
        const uint32_t w10 = lds32(aw + kM1Bytes), w11 = lds32(aw + kM1Bytes + kDwBytes);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b >= nblk) break;
          const uint4 xv = lds128(xg + b * 8 * kXP + i * 64);
          const uint4 cq = lds128(qg + b * 4 * 16 + i * (MT / 2) * 16);
          float c[4] = {__uint_as_float(cq.x), __uint_as_float(cq.y), __uint_as_float(cq.z),
                        __uint_as_float(cq.w)};
          float c1[4] = {c[0], c[1], c[2], c[3]};
          if (ZP) {
            // sum (u - z) x' = sum (u - 8) x' + (8 - z) Sx: the zero-point enters the C operand
            // per (row, token)
            const uint2 sx = lds64(sg + b * 4 * 8 + i * (MT / 2) * 8);
            const float sx0 = __uint_as_float(sx.x), sx1 = __uint_as_float(sx.y);
            float dz[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
              dz[r] = static_cast<float>(8 - static_cast<int>((zw[r][i >> 2] >> (8 * (i & 3))) & 0xFFu));
            c[0] = fmaf(dz[0], sx0, c[0]); c[1] = fmaf(dz[0], sx1, c[1]);
            c[2] = fmaf(dz[1], sx0, c[2]); c[3] = fmaf(dz[1], sx1, c[3]);
            c1[0] = fmaf(dz[2], sx0, c1[0]); c1[1] = fmaf(dz[2], sx1, c1[1]);
            c1[2] = fmaf(dz[3], sx0, c1[2]); c1[3] = fmaf(dz[3], sx1, c1[3]);
          }
          float p0[4], p1[4];
          mma_nib(p0, w00, w01, xv.x, xv.y, c, e1024);
          mma_nib(p1, w10, w11, xv.x, xv.y, c1, e1024);
          mma_nib(p0, w00 >> 8, w01 >> 8, xv.z, xv.w, p0, e1024);
          mma_nib(p1, w10 >> 8, w11 >> 8, xv.z, xv.w, p1, e1024);
          const float s0 = scale_of(sw[0], i), s1 = scale_of(sw[1], i);
          const float s2 = scale_of(sw[2], i), s3 = scale_of(sw[3], i);
          acc[b][0][0] = fmaf(s0, p0[0], acc[b][0][0]);
          acc[b][0][1] = fmaf(s0, p0[1], acc[b][0][1]);
          acc[b][0][2] = fmaf(s1, p0[2], acc[b][0][2]);
          acc[b][0][3] = fmaf(s1, p0[3], acc[b][0][3]);
          acc[b][1][0] = fmaf(s2, p1[0], acc[b][1][0]);
          acc[b][1][1] = fmaf(s2, p1[1], acc[b][1][1]);
          acc[b][1][2] = fmaf(s3, p1[2], acc[b][1][2]);
          acc[b][1][3] = fmaf(s3, p1[3], acc[b][1][3]);
        }
      }
    }
    const bool last = dflags & kDescLast;
    int sp_last = 0, tile_last = 0;     // the unit's K split and tile id (split-K epilogue)
    if (last) {
      if (A.splits > 1) {
        const int4 d1 = *reinterpret_cast<const int4*>(sp8 + kDescOff + 16);   // before the slot is freed
        sp_last = d1.y;
        tile_last = d1.z;
      }
      // undo the activation rows' power-of-two exponents (token columns 2tq, 2tq + 1 of each
      // block; the multipliers travel with the block, so no global load waits behind the stream)
      const float* mul = reinterpret_cast<const float*>(sp8 + kActOff + kMOff);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int t0 = b * 8 + 2 * tq;
        const float m0 = t0 < mt ? mul[t0] : 0.f;
        const float m1 = t0 + 1 < mt ? mul[t0 + 1] : 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          acc[b][i][0] *= m0; acc[b][i][2] *= m0;
          acc[b][i][1] *= m1; acc[b][i][3] *= m1;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (!last) continue;

    // --------------------------- epilogue (last stage of a unit) ---------------------------
    const int64_t r0 = static_cast<int>(d0.x);
    const int nt = static_cast<int>(d0.z);
    // k-part hand-over: the k-part 1 warp of each m-block stores its sums (buffer of this unit's
    // parity: the other k-part reads it before it reaches the next unit's meeting point)
    float4* rb = red + upar * (4 * NB * 2 * 32);
    if (kp == 1) {
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < 2; ++i)
          rb[((mb * NB + b) * 2 + i) * 32 + lane] = make_float4(acc[b][i][0], acc[b][i][1], acc[b][i][2], acc[b][i][3]);
    }
    upar ^= 1;
    if (!epi_sync()) return;
    if (kp == 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float4 v = rb[((mb * NB + b) * 2 + i) * 32 + lane];
          acc[b][i][0] += v.x; acc[b][i][1] += v.y; acc[b][i][2] += v.z; acc[b][i][3] += v.w;
        }
    }
    if (A.splits == 1) {
      // straight from registers: the k-part 0 thread holds rows rlo / rhi of both tiles for tokens
      // 2tq, 2tq + 1 of each block
      if (kp == 0) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int t0 = b * 8 + 2 * tq;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            if (gelu) {
              const int Nh = A.N >> 1;
              const int j = nt * kHalf + 16 * mb + 8 * i + gid;
              if (j < Nh) {
                if (t0 < mt)
                  A.out[(r0 + t0) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][i][0]) * acc[b][i][2]);
                if (t0 + 1 < mt)
                  A.out[(r0 + t0 + 1) * Nh + j] = f32_to_bf16_bits(gelu_tanh(acc[b][i][1]) * acc[b][i][3]);
              }
            } else {
              const int nlo = nt * kBN + 32 * mb + 16 * i + gid, nhi = nlo + 8;
              if (t0 < mt) {
                if (nlo < A.N) A.out[(r0 + t0) * A.N + nlo] = f32_to_bf16_bits(acc[b][i][0]);
                if (nhi < A.N) A.out[(r0 + t0) * A.N + nhi] = f32_to_bf16_bits(acc[b][i][2]);
              }
              if (t0 + 1 < mt) {
                if (nlo < A.N) A.out[(r0 + t0 + 1) * A.N + nlo] = f32_to_bf16_bits(acc[b][i][1]);
                if (nhi < A.N) A.out[(r0 + t0 + 1) * A.N + nhi] = f32_to_bf16_bits(acc[b][i][3]);
              }
            }
          }
        }
      }
    } else {
      // split-K: float32 partials through shared memory, then the last pipeline to finish its
      // part of the tile reduces them in split order (and applies the GELU gate)
      if (kp == 0) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int t0 = b * 8 + 2 * tq;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int rl = trow[2 * i], rh = trow[2 * i + 1];
            ep[t0 * kEpPitch + rl] = acc[b][i][0];
            ep[(t0 + 1) * kEpPitch + rl] = acc[b][i][1];
            ep[t0 * kEpPitch + rh] = acc[b][i][2];
            ep[(t0 + 1) * kEpPitch + rh] = acc[b][i][3];
          }
        }
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
        int is_last = 0;
        if (!flags[0]) {
          const int prev = atomicAdd(&A.counters[tile_last], 1);
          is_last = (prev == A.splits - 1);
          if (is_last) A.counters[tile_last] = 0;
        }
        flags[1] = is_last;
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
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[b][i][q] = 0.f;
  }
}

// Preparation pass: one warp per routed row r (row r of `a`, or row a_row_of_pair[r] / k_div,
// checked).  The row belongs to token block blk[e] + (r - off[e]) / MT of its expert e, at slot
// (r - off[e]) % MT (a dense linear: block r / MT).  Pass 1 finds the row's largest finite |x|
// and its exponent f (largest in [2^14, 2^15)); pass 2 writes, per 256-k block of the row, lane
// l's 8 elements 8l..8l+7 as fp16 pairs (x0, x4), (x1, x5)/16, (x2, x6), (x3, x7)/16 (scaled by
// 2^f) into the block's record of that stage, and the correction of group l / 4,
// c = -(1032 * (sum of the first and third pairs) + 1152 * (sum of the second and fourth)) summed
// over its 4 lanes (from the stored fp16 values), into components (slot & 1) and (slot & 1) + 2
// of the row pair's quad.  Elements past K are written as zero, up to the end of the last stage.
// Every stage's record also carries the row's multiplier 2^-f, so that a unit's epilogue finds
// it next to its last stage.  The zero-point variant also stores each group's sum of the row's x'
// values, Sx = (first + third pairs) + 16 (second + fourth pairs), into the row pair's Sx slot.
template <int MT, int GS, bool ZP>
__global__ void __launch_bounds__(256)
stream_prep_kernel(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair, int k_div,
                   int64_t a_rows, int64_t rows, int K, const int32_t* __restrict__ offsets, int E,
                   uint8_t* __restrict__ xw, int n_stages, int64_t n_blocks, int32_t* __restrict__ counters,
                   int n_counters, int32_t* dev_status) {
  constexpr int kRec = rec_bytes(MT, GS, ZP);
  constexpr int kXP = rec_xp(GS);
  constexpr int kQOff = rec_qoff(MT, GS);
  constexpr int kMOff = rec_moff(MT, GS);
  constexpr int kSOff = rec_soff(MT, GS);
  constexpr int kBPS = GS / kBoxG;               // 256-k blocks per stage
  extern __shared__ int prep_smem[];
  int* offs = prep_smem;                          // [E + 1]
  int* blk = prep_smem + (E + 1);                 // [E + 1]
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = K >> 3;                          // 8-element chunks in the row
  const int nblk = n_stages * kBPS;               // 256-k blocks written (zeros past K)
  // The GEMM after this pass may launch only once the kernels before the pass have completed
  // (it reads the routing and starts its weight stream before waiting for this pass).
  pdl_wait();
  pdl_trigger();
  // the GEMM's split-K arrival counters start at zero whatever the workspace held before
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_counters; i += gridDim.x * blockDim.x)
    counters[i] = 0;
  if (offsets) {
    // per-expert row offsets and first token blocks (the GEMM checks the offsets and reports)
    if (threadIdx.x < 32) {
      int brun = 0;
      for (int base = 0; base < E; base += 32) {
        const int e = base + lane;
        int nb = 0;
        if (e < E) {
          const int o0 = offsets[e], o1 = offsets[e + 1];
          offs[e] = o0;
          nb = o1 > o0 ? (o1 - o0 + MT - 1) / MT : 0;
          if (e == E - 1) offs[E] = o1;
        }
        int incl = nb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < E) blk[e] = brun + incl - nb;
        brun += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();
  }
  for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    int64_t src = r;
    if (a_row_of_pair) {
      src = __ldg(a_row_of_pair + r) / k_div;
      if (src < 0 || src >= a_rows) {
        if (lane == 0) set_status(dev_status, W4_ERR_INVALID_ARG);
        src = 0;
      }
    }
    int64_t b;
    int slot;
    if (offsets) {
      int lo = 0, hi = E - 1;                     // largest e with offs[e] <= r
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] <= r) lo = mid; else hi = mid - 1;
      }
      const int64_t local = r - offs[lo];
      // offsets out of range (the GEMM reports them): nothing is written outside the records
      if (local < 0 || r >= offs[E]) continue;
      b = blk[lo] + local / MT;
      if (b >= n_blocks) continue;
      slot = static_cast<int>(local % MT);
    } else {
      b = r / MT;
      slot = static_cast<int>(r % MT);
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
    uint8_t* rec0 = xw + b * n_stages * kRec;
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
        const float sa = (f0.x + f0.y) + (f2.x + f2.y), sb = (f1.x + f1.y) + (f3.x + f3.y);
        float part = 1032.f * sa + 1152.f * sb;
        float sxp = ZP ? sa + 16.f * sb : 0.f;
        uint8_t* rec = rec0 + static_cast<int64_t>(j / kBPS) * kRec;
        const int sub = j % kBPS;                 // 256-k block within the stage
        *reinterpret_cast<uint4*>(rec + slot * kXP + (sub * 32 + lane) * 16) = make_uint4(h[0], h[1], h[2], h[3]);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if (ZP) {
          sxp += __shfl_xor_sync(0xffffffffu, sxp, 1);
          sxp += __shfl_xor_sync(0xffffffffu, sxp, 2);
        }
        if ((lane & 3) == 0) {
          const int gi = sub * kBoxG + (lane >> 2);
          float* q = reinterpret_cast<float*>(rec + kQOff + (gi * (MT / 2) + (slot >> 1)) * 16) + (slot & 1);
          q[0] = -part;
          q[2] = -part;
          if (ZP) reinterpret_cast<float*>(rec + kSOff + (gi * (MT / 2) + (slot >> 1)) * 8)[slot & 1] = sxp;
        }
      }
    }
    for (int j = lane; j < n_stages; j += 32)
      *reinterpret_cast<float*>(rec0 + static_cast<int64_t>(j) * kRec + kMOff + slot * 4) = pow2f(-f);
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

// Scales [rows_total, kg] bf16 as a 2-D tensor (kg % 8 == 0): box = GS groups x 64 rows.
static bool encode_scales_map(CUtensorMap* m, const uint16_t* scales, int64_t rows_total, int kg, int GS) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kg), static_cast<cuuint64_t>(rows_total)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kg) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(GS), static_cast<cuuint32_t>(w4::kHalf)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Ring depth and offsets for one launch: each of the CTA's two pipelines gets half of the shared
// memory left next to the unit table, with as many slots (up to kMaxStages) as fit.
static w4::Layout make_layout(int MT, int GS, int scale_mode, int kg, int E, bool split, bool zp) {
  w4::Layout L{};
  L.sc_bytes = scale_mode == w4::kScaleTma ? 2 * w4::kHalf * GS * 2
             : scale_mode == w4::kScaleBlock ? 2 * w4::kHalf * kg * 2 : 0;
  L.slot_bytes = (w4::slot_sc_off(MT, GS, zp) + L.sc_bytes + 1023) & ~1023;
  const int table_bytes = (E + 1) * 12;
  const int ep_bytes = split ? MT * w4::kEpPitch * 4 : 0;
  const int red_bytes = 2 * 4 * (MT / 8) * 2 * 32 * 16;
  const int budget = ((w4::kSmemPerCta - 1024 - table_bytes) / w4::kPipes) & ~1023;   // per pipeline
  const int fixed = ep_bytes + red_bytes + (2 * w4::kMaxStages + 1) * 8 + 16 + 128;
  int S = (budget - fixed) / L.slot_bytes;
  if (S > w4::kMaxStages) S = w4::kMaxStages;
  L.stages = S;
  int off = S * L.slot_bytes;
  L.ep_off = split ? off : -1;
  off += ep_bytes;
  L.red_off = off;                               // (16-byte aligned: slots are 1 KB, ep 16 B multiples)
  off += red_bytes;
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
  int splits, stages_per_split, n_tiles, MT, GS, n_stages;
};

static StreamPlan plan_stream(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count) {
  StreamPlan p;
  const int kg = K / 32;
  // token block: 8 rows when experts hold few rows on average (keeps the activation record small
  // and the stages long), else 16
  p.MT = (rows <= 6LL * E) ? 8 : 16;
  p.GS = p.MT == 8 ? 16 : 8;
  p.n_stages = (kg + p.GS - 1) / p.GS;
  p.n_tiles = (epi == W4_EPI_GELU_GATE) ? ((N / 2) + w4::kHalf - 1) / w4::kHalf
                                        : (N + w4::kBN - 1) / w4::kBN;
  p.splits = 1;
  // Split K into as many parts as keep all units within one wave of the pipelines (long units
  // stream better than many short ones, and a second wave of split units costs more than it
  // saves), with at least two stages per part and float32 partials below ~1/8 of the weight
  // bytes.  Grouped calls count the token blocks the most spread-out routing can produce: at
  // most one per row, and at most one per expert plus one per MT rows.
  const int64_t ntb = dense ? (rows + p.MT - 1) / p.MT
                            : std::min<int64_t>(rows, static_cast<int64_t>(E) + rows / p.MT);
  const int64_t units = std::max<int64_t>(1, ntb * p.n_tiles);
  const double wbytes = static_cast<double>(E) * N * K * 0.5625;
  int64_t sp = static_cast<int64_t>(w4::kPipes) * sm_count / units;
  sp = std::min<int64_t>(sp, p.n_stages / 2);
  while (sp > 1 && static_cast<double>(sp) * rows * N * 4.0 > wbytes / 8.0) --sp;
  p.splits = sp > 1 ? static_cast<int>(sp) : 1;
  p.stages_per_split = (p.n_stages + p.splits - 1) / p.splits;
  p.splits = (p.n_stages + p.stages_per_split - 1) / p.stages_per_split;
  return p;
}

// Workspace: the prepared records [token block][stage][rec_bytes] (256-byte aligned); with
// split-K then the per-tile arrival counters (cleared by every launch) and the float32 partials
// [splits, rows, N].
static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// token blocks: at most one per row, and at most one per expert holding rows plus one per MT rows
static int64_t block_capacity(int64_t rows, int MT, int E, bool dense) {
  if (dense) return (rows + MT - 1) / MT;
  return std::min<int64_t>(rows, rows / MT + std::min<int64_t>(E, rows));
}

static size_t prep_bytes(const StreamPlan& p, int64_t rows, int E, bool dense, bool zp) {
  return align256(static_cast<size_t>(block_capacity(rows, p.MT, E, dense)) * p.n_stages *
                  w4::rec_bytes(p.MT, p.GS, zp));
}

// one arrival counter per (expert, token block, weight tile)
static size_t counters_bytes(const StreamPlan& p, int64_t rows, int E, bool dense) {
  return align256(static_cast<size_t>(block_capacity(rows, p.MT, E, dense) * p.n_tiles) * sizeof(int32_t));
}

size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count,
                                 bool zp) {
  if (rows <= 0) return 0;
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  size_t b = prep_bytes(p, rows, E, dense, zp);
  if (p.splits > 1)
    b += counters_bytes(p, rows, E, dense) + static_cast<size_t>(p.splits) * rows * N * sizeof(float);
  return b;
}

template <int MT, int GS, bool GELU, int SCALE, bool ZP>
static w4_status launch_one(const CUtensorMap& tmap, const CUtensorMap& smap, const w4::StreamArgs& A,
                            int sm_count, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel<MT, GS, GELU, SCALE, ZP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, w4::kSmemPerCta) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  return launch_pdl(w4::stream_gemm_kernel<MT, GS, GELU, SCALE, ZP>, dim3(sm_count), dim3(w4::kThreads),
                    A.L.total, stream, tmap, smap, A) == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

template <int MT, int GS, bool GELU>
static w4_status launch_scale(int scale_mode, bool zp, const CUtensorMap& tmap, const CUtensorMap& smap,
                              const w4::StreamArgs& A, int sm_count, cudaStream_t stream) {
  if (zp) return launch_one<MT, GS, GELU, w4::kScaleLdg, true>(tmap, smap, A, sm_count, stream);
  if (scale_mode == w4::kScaleTma) return launch_one<MT, GS, GELU, w4::kScaleTma, false>(tmap, smap, A, sm_count, stream);
  if (scale_mode == w4::kScaleBlock) return launch_one<MT, GS, GELU, w4::kScaleBlock, false>(tmap, smap, A, sm_count, stream);
  return launch_one<MT, GS, GELU, w4::kScaleLdg, false>(tmap, smap, A, sm_count, stream);
}

template <int MT, int GS>
static cudaError_t launch_prep(bool zp, dim3 grid, size_t smem, cudaStream_t stream, const uint16_t* a,
                               const int32_t* a_row_of_pair, int kd, int64_t a_rows, int64_t rows, int K,
                               const int32_t* offsets, int E, uint8_t* xw, int n_stages, int64_t n_blocks,
                               int32_t* counters, int n_counters, int32_t* dev_status) {
  if (zp)
    return launch_pdl(w4::stream_prep_kernel<MT, GS, true>, grid, dim3(256), smem, stream, a, a_row_of_pair, kd,
                      a_rows, rows, K, offsets, E, xw, n_stages, n_blocks, counters, n_counters, dev_status);
  return launch_pdl(w4::stream_prep_kernel<MT, GS, false>, grid, dim3(256), smem, stream, a, a_row_of_pair, kd,
                    a_rows, rows, K, offsets, E, xw, n_stages, n_blocks, counters, n_counters, dev_status);
}

w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count, uint64_t wait_ns, int stall_after,
                                const uint8_t* zeros, int group) {
  const bool dense = (offsets == nullptr);
  const bool zp = zeros != nullptr;
  int gshift = 0;
  while ((32 << gshift) < group) ++gshift;
  if ((32 << gshift) != group || K % group) return W4_ERR_INVALID_ARG;   // (callers check first)
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  w4::StreamArgs A{};
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32; A.rows = rows; A.epi = epi; A.out = out;
  A.zeros = zeros; A.gshift = gshift; A.kgs = K / group;
  A.splits = p.splits; A.stages_per_split = p.stages_per_split; A.n_tiles = p.n_tiles;
  A.n_stages = p.n_stages;
  A.dev_status = dev_status;
  A.wait_ns = wait_ns ? wait_ns : w4::kWaitLimitNs;
  A.stall_after = stall_after;
  {
    // grouped calls whose experts' weights fit in half of L2 (a few decode tokens): prefetch
    // every stage at the start (a dense K = 4096 GEMV got slower with it: its ring's first loads
    // queue behind the prefetches)
    const double touched = static_cast<double>(std::min<int64_t>(E, rows)) * N * K * 0.5625;
    A.pf_all = !dense && touched <= 64.0 * (1 << 20);
  }
  // Scale staging: 2-D TMA when a scale row is a whole number of 16-byte chunks; else the tile's
  // contiguous 64-row scale blocks by bulk copy when they are 16-byte aligned and small; else
  // direct loads.
  const bool s16 = (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
  int scale_mode;
  if (zp || group != 32) {
    scale_mode = w4::kScaleLdg;            // variants: scales (and zero-points) by direct loads
  } else if (A.kg % 8 == 0 && s16) {
    scale_mode = w4::kScaleTma;
  } else if (A.kg % 2 == 0 && A.kg <= w4::kBlockMaxKg && N % 8 == 0 && s16 &&
             (epi == W4_EPI_GELU_GATE ? (N / 2) % w4::kHalf == 0 : N % w4::kBN == 0)) {
    // (whole tiles only: the 64-row blocks are plain bulk copies and must stay inside the array)
    scale_mode = w4::kScaleBlock;
  } else {
    scale_mode = w4::kScaleLdg;
  }
  A.L = make_layout(p.MT, p.GS, scale_mode, A.kg, E, p.splits > 1, zp);
  if (A.L.stages < 2) return W4_ERR_UNSUPPORTED;
  if (rows == 0) return W4_OK;
  const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count, zp);
  if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  A.xw = wsb;
  if (p.splits > 1) {
    uint8_t* cbase = wsb + prep_bytes(p, rows, E, dense, zp);
    const size_t cb = counters_bytes(p, rows, E, dense);
    A.counters = reinterpret_cast<int32_t*>(cbase);
    A.partial = reinterpret_cast<float*>(cbase + cb);
    // (the preparation pass clears the arrival counters)
  }
  {
    const int kd = k_div > 0 ? k_div : 1;
    const int64_t a_rows = a_row_of_pair ? rows / kd : rows;
    const int64_t wblocks = (rows + 7) / 8;
    const int grid = static_cast<int>(wblocks < 16LL * sm_count ? wblocks : 16LL * sm_count);
    const int n_counters =
        p.splits > 1 ? static_cast<int>(counters_bytes(p, rows, E, dense) / sizeof(int32_t)) : 0;
    const size_t psmem = dense ? 0 : static_cast<size_t>(E + 1) * 2 * sizeof(int);
    const int64_t nb = block_capacity(rows, p.MT, E, dense);
    const int32_t* offs = dense ? nullptr : offsets;
    const cudaError_t e = p.MT == 8
        ? launch_prep<8, 16>(zp, dim3(grid), psmem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offs, E, wsb,
                             p.n_stages, nb, A.counters, n_counters, dev_status)
        : launch_prep<16, 8>(zp, dim3(grid), psmem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offs, E, wsb,
                             p.n_stages, nb, A.counters, n_counters, dev_status);
    if (e != cudaSuccess) return W4_ERR_CUDA;
  }
  CUtensorMap tmap, smap;
  std::memset(&smap, 0, sizeof(smap));
  if (!encode_codes_map(&tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  if (scale_mode == w4::kScaleTma &&
      !encode_scales_map(&smap, scales, static_cast<int64_t>(E) * N, A.kg, p.GS))
    return W4_ERR_CUDA;
  const bool gelu = A.epi == W4_EPI_GELU_GATE;
  if (p.MT == 8)
    return gelu ? launch_scale<8, 16, true>(scale_mode, zp, tmap, smap, A, sm_count, stream)
                : launch_scale<8, 16, false>(scale_mode, zp, tmap, smap, A, sm_count, stream);
  return gelu ? launch_scale<16, 8, true>(scale_mode, zp, tmap, smap, A, sm_count, stream)
              : launch_scale<16, 8, false>(scale_mode, zp, tmap, smap, A, sm_count, stream);
}
