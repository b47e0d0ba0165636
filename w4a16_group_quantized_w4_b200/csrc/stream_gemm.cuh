// Weight-streaming W4A16 GEMM: device code shared by its own kernels (stream_gemm.cu) and the
// fused MoE decode kernel (fused.cu).  The design notes are at the top of stream_gemm.cu.
#pragma once

#include <cudaTypedefs.h>

#include <type_traits>

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
// ring at p * pipe_bytes, its k-part hand-over buffer, barriers and flags after the ring; then the
// unit table.
struct Layout {
  int stages;
  int slot_bytes;            // one slot (multiple of 1024)
  int sc_bytes;              // scale bytes per slot
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
  // Hand-over inside one kernel (the fused MoE decode kernel, which instantiates the body with
  // HO = true; unused otherwise): the producers copy a token block's records only once
  // act_ready[block] has reached the block's row count, and every finished (block, weight tile)
  // adds one to tile_done[block] once its outputs are written.
  const int32_t* act_ready;
  int32_t* tile_done;
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
// 16 bytes (read every stage), {expert, K split, tile id, token block} in the second (read only by
// the epilogue of a split-K or handed-over unit and by the direct-load scale mode).  The tile id numbers the (expert, token
// block, weight tile) triples 0.. densely; the split-K arrival counters are indexed by it.
enum : int { kDescFirst = 1, kDescLast = 2, kDescDone = 4 };
struct __align__(16) StageDesc {
  int r0;
  int g;
  int nt;
  int bits;
  int e, sp, tile, blk;
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

struct NoPreWork {
  __device__ void operator()(const int*, const int*, int, int) const {}
};

// The kernel's body (stream_gemm_kernel, and two phases of the fused MoE decode kernel): smem_raw
// is the dynamic shared memory of the CTA.  HO: the in-kernel hand-over through A.act_ready /
// A.tile_done is compiled in.  SPL: the epilogue for units without a K split (0), with one (1),
// or either, chosen by A.splits at run time (2); the stand-alone kernel is instantiated per case
// so that each carries only the epilogue it runs.  pre(offs, blk, w, n) runs on the n = 16 compute warps (w = 0..15)
// once the unit table is built and before they consume the first stage, while the producers
// already stream weights: offs / blk are the table's per-expert row offsets and first token
// blocks (shared memory).  It may use warp-level synchronisation only.
template <int MT, int GS, bool GELU, int SCALE, bool ZP, int SPL = 2, bool HO = false, typename Pre = NoPreWork>
__device__ __forceinline__ void stream_gemm_body(const CUtensorMap& tmap_codes, const CUtensorMap& tmap_scales,
                                                 const StreamArgs& A, uint8_t* smem_raw, const Pre& pre = Pre{}) {
  constexpr int kActOff = slot_act_off(GS);
  constexpr int kDescOff = slot_desc_off(MT, GS, ZP);
  constexpr int kScOff = slot_sc_off(MT, GS, ZP);
  constexpr int kRec = rec_bytes(MT, GS, ZP);
  constexpr int kSOff = rec_soff(MT, GS);
  constexpr int kXP = rec_xp(GS);
  constexpr int kQOff = rec_qoff(MT, GS);
  constexpr int kMOff = rec_moff(MT, GS);
  constexpr int NB = MT / 8;                    // token blocks of 8 (the MMA's n)
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
    struct DeferredPlain { uint8_t* dst; const uint8_t* src; uint32_t bytes; uint64_t* bar; };
    struct DeferredHO { uint8_t* dst; const uint8_t* src; uint32_t bytes; uint64_t* bar; int blk, need; };
    using Deferred = typename std::conditional<HO, DeferredHO, DeferredPlain>::type;
    Deferred def[2 * kMaxStages];
    int ndef = 0;
    bool waited = false;
    // In-kernel hand-over: wait (bounded) until the block's rows are all written.  A wait that runs
    // out reports W4_ERR_TIMEOUT and the copy goes ahead (the slot accounting stays intact, so
    // the kernel still ends normally), and no later wait is made.
    int ready_blk = -1;
    bool ready_gave_up = false;
    auto ready_wait = [&](int b, int need) {
      if (!HO || !A.act_ready || b == ready_blk || ready_gave_up) return;
      if (!wait_count(A.act_ready + b, need, A.wait_ns)) {
        set_status(A.dev_status, W4_ERR_TIMEOUT);
        ready_gave_up = true;
      }
      fence_proxy_async_global();
      ready_blk = b;
    };
    auto act_copy = [&](uint8_t* dst, const uint8_t* src, uint32_t bytes, uint64_t* bar, int b, int need) {
      if (waited) {
        ready_wait(b, need);
        bulk_g2s(dst, src, bytes, bar);
      } else {
        if constexpr (HO) def[ndef++] = Deferred{dst, src, bytes, bar, b, need};
        else def[ndef++] = Deferred{dst, src, bytes, bar};
      }
    };
    auto flush = [&]() {
      if (waited) return;
      pdl_wait();
      waited = true;
      for (int i = 0; i < ndef; ++i) {
        if constexpr (HO) ready_wait(def[i].blk, def[i].need);
        bulk_g2s(def[i].dst, def[i].src, def[i].bytes, def[i].bar);
      }
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
        dsc.blk = HO ? U.blk : 0;
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
          act_copy(sl + kActOff, rec, kRec, &full[slot], U.blk, U.mt);
        } else {
          act_copy(sl + kActOff, rec, U.mt * kXP, &full[slot], U.blk, U.mt);
          act_copy(sl + kActOff + kQOff, rec + kQOff, kRec - kQOff, &full[slot], U.blk, U.mt);
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
  pre(offs, blk, warp_all, kPipes * kWarps);
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
    int sp_last = 0, tile_last = 0, blk_last = 0;   // the unit's K split, tile id, token block
    if (last) {
      if ((SPL == 2 ? A.splits > 1 : SPL == 1) || HO) {
        const int4 d1 = *reinterpret_cast<const int4*>(sp8 + kDescOff + 16);   // before the slot is freed
        sp_last = d1.y;
        tile_last = d1.z;
        blk_last = d1.w;
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
    if (SPL == 2 ? A.splits == 1 : SPL == 0) {
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
      if (HO && A.tile_done) {
        // hand-over: once the warps have met, one thread makes their outputs visible GPU-wide
        // (a fence after the meeting covers every write ordered before it) and moves the count
        if (!epi_sync()) return;
        if (warp == 0 && lane == 0) {
          __threadfence();
          atomicAdd(A.tile_done + blk_last, 1);
        }
      }
    } else {
      // split-K: each K part writes its float32 partials straight from registers; the last
      // pipeline to finish its part of the tile reduces them in split order (and applies the
      // GELU gate).  One meeting puts every warp's partials before the thread that counts the
      // arrival (its fence after the meeting covers them all), a second passes the verdict on.
      const int ctid = warp * 32 + lane;
      const int Nh = A.N >> 1;
      if (kp == 0 && !flags[0]) {
        float* pbase = A.partial + (static_cast<int64_t>(sp_last) * A.rows + r0) * A.N;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          // partial columns of this thread's rows (GELU: rows 0..63 gate j, 64..127 up j)
          int nl, nh;
          bool okl, okh;
          if (gelu) {
            const int j = nt * kHalf + 16 * mb + 8 * i + gid;
            okl = okh = j < Nh;
            nl = j;
            nh = Nh + j;
          } else {
            nl = nt * kBN + trow[2 * i];
            nh = nt * kBN + trow[2 * i + 1];
            okl = nl < A.N;
            okh = nh < A.N;
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const int t0 = b * 8 + 2 * tq;
            if (t0 < mt) {
              if (okl) pbase[static_cast<int64_t>(t0) * A.N + nl] = acc[b][i][0];
              if (okh) pbase[static_cast<int64_t>(t0) * A.N + nh] = acc[b][i][2];
            }
            if (t0 + 1 < mt) {
              if (okl) pbase[static_cast<int64_t>(t0 + 1) * A.N + nl] = acc[b][i][1];
              if (okh) pbase[static_cast<int64_t>(t0 + 1) * A.N + nh] = acc[b][i][3];
            }
          }
        }
      }
      if (!epi_sync()) return;
      if (ctid == 0) {
        int is_last = 0;
        if (!flags[0]) {
          __threadfence();
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
      // (flags[1] is next written two meetings into the next split unit, after every warp has
      // read it here)
      if (HO && A.tile_done) {
        if (!epi_sync()) return;
        if (flags[1] && ctid == 0) {
          __threadfence();
          atomicAdd(A.tile_done + blk_last, 1);
        }
      }
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
// The pass's body (stream_prep_kernel, and two phases of the fused MoE decode kernel); prep_smem
// holds 2 (E + 1) ints.  Any number of warps per CTA.
//
// Hand-over inside one kernel (PrepHooks, all null in the stand-alone pass): a row waits until
// src_ready[its block] reaches src_need before reading its source row (the source is written by
// an earlier phase of the same kernel), and once its records are written adds one to
// ready[its block]; row_blk[r] receives the row's token block.  INK: `a` and a_row_of_pair are
// written inside the same kernel, so they are read through L2 (not the read-only path).
struct PrepHooks {
  const int32_t* src_ready;
  int src_need;
  int32_t* ready;
  int32_t* row_blk;
  uint64_t wait_ns;
};

// Work items [wfirst, rows * nchunk) in steps of wstride, one warp each: item w is row
// w / nchunk, 256-k blocks [c * bchunk, (c + 1) * bchunk) with c = w % nchunk (every item finds
// the row's exponent over the whole row; CHUNK = false compiles whole rows only, which the
// hand-over hooks require).  offs / blk are the per-expert row offsets and first token blocks
// (grouped), held in shared memory.
template <int MT, int GS, bool ZP, bool INK, bool CHUNK = false>
__device__ __forceinline__ void stream_prep_rows(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair,
                                                 int k_div, int64_t a_rows, int64_t rows, int K, bool grouped,
                                                 const int* offs, const int* blk, int E, uint8_t* __restrict__ xw,
                                                 int n_stages, int64_t n_blocks, int32_t* dev_status,
                                                 const PrepHooks& hk, int64_t wfirst, int64_t wstride,
                                                 int bchunk = 1 << 20) {
  constexpr int kRec = rec_bytes(MT, GS, ZP);
  constexpr int kXP = rec_xp(GS);
  constexpr int kQOff = rec_qoff(MT, GS);
  constexpr int kMOff = rec_moff(MT, GS);
  constexpr int kSOff = rec_soff(MT, GS);
  constexpr int kBPS = GS / kBoxG;               // 256-k blocks per stage
  const int lane = threadIdx.x & 31;
  const int nv = K >> 3;                          // 8-element chunks in the row
  const int nblk = n_stages * kBPS;               // 256-k blocks written (zeros past K)
  if (bchunk > nblk) bchunk = nblk;
  const int nchunk = CHUNK ? (nblk + bchunk - 1) / bchunk : 1;
  for (int64_t w = wfirst; w < rows * nchunk; w += wstride) {
    const int64_t r = CHUNK ? w / nchunk : w;
    const int jb0 = CHUNK ? static_cast<int>(w - r * nchunk) * bchunk : 0;   // this item's blocks
    const int jb1 = !CHUNK ? nblk : (jb0 + bchunk < nblk ? jb0 + bchunk : nblk);
    int64_t src = r;
    if (a_row_of_pair) {
      src = (INK ? __ldcg(a_row_of_pair + r) : __ldg(a_row_of_pair + r)) / k_div;
      if (src < 0 || src >= a_rows) {
        if (lane == 0) set_status(dev_status, W4_ERR_INVALID_ARG);
        src = 0;
      }
    }
    int64_t b;
    int slot;
    if (grouped) {
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
    if (hk.row_blk && lane == 0) hk.row_blk[r] = static_cast<int32_t>(b);
    if (hk.src_ready) {
      bool ok = true;
      if (lane == 0) ok = wait_count(hk.src_ready + b, hk.src_need, hk.wait_ns);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) && lane == 0) set_status(dev_status, W4_ERR_TIMEOUT);
    }
    const uint4* row = reinterpret_cast<const uint4*>(a + src * K);
    auto ld_row = [&](int i) -> uint4 { return INK ? __ldcg(row + i) : __ldg(row + i); };
    // Lane l holds chunk l of up to kPB 256-k blocks at a time, all loads of a batch in flight
    // together; a row of at most kPB blocks is read once.
    uint4 v[kPB];
    uint32_t m = 0;
    for (int j0 = 0; j0 < nblk; j0 += kPB) {
#pragma unroll
      for (int t = 0; t < kPB; ++t) {
        const int i = (j0 + t) * 32 + lane;
        v[t] = i < nv ? ld_row(i) : make_uint4(0, 0, 0, 0);
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
    for (int j0 = jb0; j0 < jb1; j0 += kPB) {
      if (nblk > kPB || (CHUNK && jb0 > 0)) {    // the batch again (from L1 / L2)
#pragma unroll
        for (int t = 0; t < kPB; ++t) {
          const int i = (j0 + t) * 32 + lane;
          v[t] = i < nv && j0 + t < jb1 ? ld_row(i) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int t = 0; t < kPB; ++t) {
        const int j = j0 + t;
        if (j >= jb1) break;
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
    // the row's multiplier in every stage whose first block is this item's
    for (int j = lane; j < n_stages; j += 32)
      if (!CHUNK || (j * kBPS >= jb0 && j * kBPS < jb1))
        *reinterpret_cast<float*>(rec0 + static_cast<int64_t>(j) * kRec + kMOff + slot * 4) = pow2f(-f);
    if (hk.ready) {
      // the records are read by bulk copies (the async proxy) of other CTAs; the release is made
      // once for the warp's writes, after the warp has met
      fence_proxy_async_global();
      __syncwarp();
      if (lane == 0) {
        __threadfence();
        atomicAdd(hk.ready + b, 1);
      }
    }
  }
}

template <int MT, int GS, bool ZP, bool INK = false, bool CHUNK = false>
__device__ __forceinline__ void stream_prep_body(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair,
                                                 int k_div, int64_t a_rows, int64_t rows, int K,
                                                 const int32_t* __restrict__ offsets, int E, uint8_t* __restrict__ xw,
                                                 int n_stages, int64_t n_blocks, int32_t* __restrict__ counters,
                                                 int n_counters, int32_t* dev_status, int* prep_smem,
                                                 int bchunk = 1 << 20, const PrepHooks& hk = PrepHooks{}) {
  int* offs = prep_smem;                          // [E + 1]
  int* blk = prep_smem + (E + 1);                 // [E + 1]
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
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
          const int o0 = INK ? __ldcg(offsets + e) : offsets[e];
          const int o1 = INK ? __ldcg(offsets + e + 1) : offsets[e + 1];
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
  stream_prep_rows<MT, GS, ZP, INK, CHUNK>(a, a_row_of_pair, k_div, a_rows, rows, K, offsets != nullptr, offs, blk, E, xw,
                                    n_stages, n_blocks, dev_status, hk, blockIdx.x * wpb + (threadIdx.x >> 5),
                                    gridDim.x * wpb, bchunk);
}

}  // namespace w4

namespace w4 {
// Ends a GEMM phase inside a longer kernel: invalidates the phase's mbarriers so that their
// shared memory can be reused (called by one thread after a CTA barrier that every warp of the
// phase has reached).
__device__ __forceinline__ void stream_gemm_inval(const Layout& L, uint8_t* smem_raw) {
  uint8_t* smem0 = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  for (int p = 0; p < kPipes; ++p) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem0 + p * L.pipe_bytes + L.bar_off);
    for (int i = 0; i < 2 * L.stages + 1; ++i) mbar_inval(bars + i);
  }
}
}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host side (stream_gemm.cu): the arguments of one streaming-GEMM call, shared with the fused MoE
// decode kernel
// ---------------------------------------------------------------------------------------------
struct StreamPlan {
  int splits, stages_per_split, n_tiles, MT, GS, n_stages;
};

struct StreamCall {
  w4::StreamArgs A;         // everything but the workspace pointers and the output
  StreamPlan p;
  int scale_mode;
  CUtensorMap tmap, smap;   // codes; scales (2-D TMA scale mode only)
  int64_t n_blocks;         // token-block capacity (prepared records)
  size_t prep_bytes;        // workspace: records, then split-K counters and partials
  size_t counters_bytes;
  size_t partial_bytes;
};

// Plans the call and encodes its tensor maps (offsets == nullptr: a dense linear); allow_block
// false keeps the call off the bulk-copied scale-block mode.
w4_status w4_stream_setup(const uint32_t* codes, const uint16_t* scales, const int32_t* offsets, int E,
                          int64_t rows, int N, int K, int epi, int32_t* dev_status, int sm_count,
                          uint64_t wait_ns, int stall_after, const uint8_t* zeros, int group, StreamCall& C,
                          bool allow_block = true);
// Points the call's records, counters and partials into the workspace at ws.
void w4_stream_bind(StreamCall& C, uint8_t* ws);
