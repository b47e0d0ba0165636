// Tensor-core W4A16 grouped GEMM with the dequantised weights held in tensor memory, for many
// routed rows per weight matrix (prefill, dense linears with M >= 64).
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "What changed in vLLM's TPU backend": the grouped matmul takes a scale per 32-wide group and
// dequantises each weight tile in fast on-chip memory before the multiply; activations stay
// 16-bit.  Here the on-chip memory is the SM's tensor memory (TMEM): the dequantised weight tile
// is the A operand of tcgen05.mma straight from TMEM, so it never round-trips through shared
// memory, and the routed token rows are the B operand, staged by TMA.
//
// Decode batches (a few rows per expert) do not use this kernel: one issuing thread retires a
// tcgen05.mma about every 90-170 cycles whatever N is, so at N = 16 the MMAs alone cap a
// 128-row weight tile at about 1 KB of codes per 100 cycles per SM, below the HBM rate; the
// weight-streaming kernel (mma.sync issued by eight warps) serves them.
//
// Exactness: the tile holds fp16(s * 2^e * q), e a power of two per weight row chosen from the
// row's largest scale.  s * q has at most 11 significant bits (8 from the bf16 scale, 3 from
// |q| <= 8), which fp16 holds exactly; the activations were converted to fp16 with a
// power-of-two exponent per row (convert.cu).  The tensor core therefore forms the exact
// a * s * q, accumulates in fp32, and the epilogue multiplies by 2^-f and 2^-e (exact).
//
// Dequantisation of one code pair, exact in two instructions: lop3 puts the two 4-bit fields u
// (moved to bits 6-9 and 22-25) under the fp16 exponent of 1024, giving x = 1024 + 64u; then
// fma(x, s'', -1536 s'') = (u - 8) s' with s'' = s' / 64, s' = s * 2^e:
// x s'' = 16 s' + u s' and 1536 s'' = 24 s'.  The constant 1536 s'' = 3 s'' * 2^9 has at most
// 10 significant bits, so it is exact, and (u - 8) s' has at most 11, so the one rounding of the
// FMA is exact as well (checked exhaustively over the bf16 scales within 2^21 of the row's
// largest and all 16 codes).  With the nibble any lower in the mantissa the constant would be
// 72 s' or worse, which can carry into a 12th bit.
//
// Tile: 128 weight rows (MMA M, one TMEM lane each) x up to NMAX routed rows (MMA N) x all of K
// in stages of KSK k.  With the GELU gate the 128 weight rows are 64 gate rows and the 64 up
// rows of the same outputs, laid out over the TMEM lanes so that lane i and lane i ^ 16 hold the
// gate and up row of one output.
//
// Three rings decouple the latencies: codes (shared memory, as deep as the shared-memory budget
// allows; a slot is free again as soon as the dequant warps have read it, so only the HBM latency
// sets how many bytes must be in flight), tokens (shared memory, held until the MMAs have read
// them) and dequantised weights (TMEM slots of 128 k, held until the MMAs have read them).
//
// Roles (persistent CTA, one per SM, 16 warps):
//   warp 0       code producer: per stage, two 2-D TMA boxes of the 128 weight rows (swizzled)
//   warp 3       token producer: per stage, 2-D TMA boxes of 64 k x NMAX rows (128-byte swizzle)
//   warp 1       TMEM allocation and the MMA-issuing thread (warps 16.. add issuers when the
//                configuration splits a tile's MMAs over several threads)
//   warp 2       idle (the dequant warps read their scales from global memory, see below)
//   warps 4-7    epilogue: tcgen05.ld of the accumulator, exponents, GELU gate, bf16 stores
//   warps 8-15   dequant: codes + scales -> fp16 pairs -> tcgen05.st into the TMEM A slots.
//                Each thread owns one weight row: its exponent e comes from the conversion pass
//                (one byte per weight row, loaded a tile ahead) and its two scales per stage
//                straight from global memory through a three-stage register queue that runs
//                ahead across tiles, so no shared memory is spent on scale blocks.
// Every wait is bounded (W4_ERR_TIMEOUT in dev_status instead of a hang).
#include <cudaTypedefs.h>

#include <cstring>

#include "tcgen05.cuh"

namespace w4 {
namespace tm {

constexpr int kBM = 128;                                 // weight rows per tile (MMA M)
constexpr int kMaxKg = 128;                              // K <= 4096
constexpr int kThreads = 16 * 32;
constexpr int kMaxCStages = 16;                          // deepest code ring
constexpr int kACols = 64;                               // TMEM columns per A slot (128 k)

// Shared-memory layout, fixed per launch (offsets from the 1024-byte aligned base).
struct Lay {
  int code;                 // code ring: cst stages
  int cst;
  int stage;                // epilogue output staging: 2 x 1 KB per epilogue warp
  int sh;                   // float [2][128]: 2^-e per TMEM lane
  int bars;
  int tmem_slot;            // + abort flag
  int table;                // int table[E+1], offs[E+1]
  int total;
};

struct Args {
  const float* rowmul;      // [rows] 2^-f of each converted activation row
  const int8_t* rowexp;     // [E*N] exponent e of each weight row
  const uint16_t* scales;   // [E*N, kg]
  const int32_t* offsets;   // [E+1] or null (dense: one expert with `rows` rows)
  int E, N, K, kg, nst;     // nst = stages per tile
  int64_t rows;
  int epi;
  uint16_t* out;
  int n_tiles;              // weight tiles per expert
  int32_t* dev_status;
  int tma_out;              // 1: whole 16-token chunks leave through shared memory and TMA stores
  Lay L;
};

// NMAX routed rows per tile, stages of KSK k, TSTAGES token stages, ASLOTS TMEM slots of
// dequantised weights, NSPLIT x KSPLIT MMA-issuing threads (token-column parts x k parts).
// KSK = 256 makes every code-row request of the TMA 128 bytes long; KSK = 128 leaves room for
// 128-row token tiles.
template <int NMAX, int KSK, int TSTAGES, int ASLOTS, int NSPLIT, int KSPLIT, int ABUF, int EPIW>
struct Cfg {
  static_assert(NMAX % 32 == 0 && NMAX <= 256, "MMA N, whole 32-token epilogue groups");
  static_assert(KSK == 128 || KSK == 256, "stage width");
  static constexpr int kSubs = KSK / 64;                 // 64-k token sub-tiles per stage
  static constexpr int kHalves = KSK / 128;              // TMEM A slots per stage
  static constexpr int kCodePitch = KSK / 2;             // bytes of one code row in a stage
  static constexpr int kCodeStage = kBM * kCodePitch;
  static constexpr int kTokSub = NMAX * 128;             // one 64-k sub-tile: NMAX rows x 128 B
  static constexpr int kTokStage = kSubs * kTokSub;
  static_assert(ABUF == 1 || ABUF == 2, "accumulator buffers");
  static_assert(EPIW == 1 || EPIW == 2, "epilogue warps per TMEM lane quadrant");
  static constexpr int kIssuers = NSPLIT * KSPLIT;
  static constexpr int kEpiWarps = 4 * EPIW;
  // warps: 0-15 fixed roles, then issuers 1.., then the second epilogue warp of each quadrant
  static constexpr int kIssuerWarp0 = 16;
  static constexpr int kEpiWarp1 = 16 + kIssuers - 1;
  static constexpr int kWarps = 16 + (kIssuers - 1) + 4 * (EPIW - 1);
  static constexpr int kNS = NMAX / NSPLIT;              // token columns per issuer
  static_assert(kNS % 16 == 0, "M = 128 MMAs take N in multiples of 16");
  // accumulator (buffer ab, k part kp) at columns [(ABUF kp + ab) NMAX, ... + NMAX); A slots after
  __host__ __device__ static constexpr uint32_t acc_col(int ab, int kp) {
    return static_cast<uint32_t>((ABUF * kp + ab) * NMAX);
  }
  static constexpr int kA0 = ABUF * KSPLIT * NMAX;
  static constexpr int kColsUsed = kA0 + ASLOTS * kACols;
  static_assert(kColsUsed <= 512, "TMEM columns");
  static constexpr uint32_t kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64
                                      : kColsUsed <= 128 ? 128 : kColsUsed <= 256 ? 256 : 512;
  static constexpr int tok = 0;                          // token ring at the base
  static constexpr int code = TSTAGES * kTokStage;       // code ring after it
  // cfull, cfree (x kMaxCStages), tfull, tfree (x TSTAGES), a_ready, a_free (x ASLOTS),
  // acc_full, acc_empty, sh_full, sh_empty (x 2)
  static constexpr int nbars = 2 * kMaxCStages + 2 * TSTAGES + 2 * ASLOTS + 8;
  static_assert(kTokSub % 1024 == 0, "128-byte swizzle atoms");
};

struct Tile {
  int e, mt, nt;
  int64_t r0;
  int mrows;
};

// Tile t -> (expert, block of routed rows, weight tile); weight tiles fastest, so the CTAs
// running together share a few token blocks (each read from HBM once and then from L2 by every
// weight tile) while each expert's weight tiles are re-read once per token block.  (Token blocks
// fastest would re-read every token block once per weight tile: for the prefill gate/up GEMM,
// 1.4 MB x 11 per block, far more than the weights.)
__device__ __forceinline__ void decode_tile(const Args& A, const int* table, const int* offs,
                                            int t, int nmax, Tile& T) {
  int lo = 0, hi = A.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (table[mid] <= t) lo = mid; else hi = mid - 1;
  }
  T.e = lo;
  const int off0 = offs[lo], off1 = offs[lo + 1];
  const int local = t - table[lo];
  T.mt = local / A.n_tiles;
  T.nt = local - T.mt * A.n_tiles;
  T.r0 = off0 + static_cast<int64_t>(T.mt) * nmax;
  T.mrows = min(nmax, off1 - static_cast<int>(T.r0));
}

// global weight row of tile row r (0..127): GELU gate rows 0-63, up rows 64-127
__device__ __forceinline__ int64_t wrow(const Args& A, const Tile& T, int r) {
  int n;
  if (A.epi == W4_EPI_GELU_GATE) {
    const int j = T.nt * (kBM / 2) + (r & (kBM / 2 - 1));
    n = (r < kBM / 2) ? j : (A.N >> 1) + j;
  } else {
    n = T.nt * kBM + r;
  }
  return static_cast<int64_t>(T.e) * A.N + n;
}

// tile row held by TMEM lane l: with the GELU gate, lanes 32q + i (i < 16) hold gate rows
// 16q + i and lanes 32q + 16 + i the up rows 64 + 16q + i, so a lane and its partner l ^ 16 hold
// one output's pair (and eight consecutive lanes read eight consecutive code rows)
__device__ __forceinline__ int lane_row(int epi, int l) {
  if (epi != W4_EPI_GELU_GATE) return l;
  const int q = l >> 5, i = l & 31;
  return i < 16 ? 16 * q + i : kBM / 2 + 16 * q + (i - 16);
}

// (u - 8) * s' for the two 4-bit fields at bits 6-9 and 22-25 of v (see the file comment)
__device__ __forceinline__ uint32_t deq_pair(uint32_t v, uint32_t s2, uint32_t c2) {
  uint32_t x, y;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(x) : "r"(v), "r"(0x03C003C0u), "r"(0x64006400u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(y) : "r"(x), "r"(s2), "r"(c2));
  return y;
}

// one code word (eight consecutive k, layout L1: nibble j = element j) -> four fp16 pairs = four
// TMEM columns, in the k order 0, 4, 1, 5, 2, 6, 3, 7 that the conversion pass gives the tokens
__device__ __forceinline__ void deq_word(uint32_t w, uint32_t s2, uint32_t c2, uint32_t* o) {
  o[0] = deq_pair(w << 6, s2, c2);   // elements 0, 4 (bits 0-3, 16-19)
  o[1] = deq_pair(w << 2, s2, c2);   // elements 1, 5 (bits 4-7, 20-23)
  o[2] = deq_pair(w >> 2, s2, c2);   // elements 2, 6 (bits 8-11, 24-27)
  o[3] = deq_pair(w >> 6, s2, c2);   // elements 3, 7 (bits 12-15, 28-31)
}

// s'' = s * 2^(e-6) and c = -1536 s'' as fp16 pairs
__device__ __forceinline__ void scale_pair(uint32_t s16, float smul, uint32_t& s2, uint32_t& c2) {
  const __half sh = __float2half_rn(bf16_lo_to_f32(s16) * smul);
  const __half ch = __hmul(sh, __float2half_rn(-1536.f));
  const __half2 a = __halves2half2(sh, sh), b = __halves2half2(ch, ch);
  s2 = *reinterpret_cast<const uint32_t*>(&a);
  c2 = *reinterpret_cast<const uint32_t*>(&b);
}


template <int NMAX, int KSK, int TSTAGES, int ASLOTS, int NSPLIT, int KSPLIT, int ABUF, int EPIW>
__global__ void __launch_bounds__(32 * (16 + (NSPLIT * KSPLIT - 1) + 4 * (EPIW - 1)), 1)
tm_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
               const __grid_constant__ CUtensorMap tmap_tok,
               const __grid_constant__ CUtensorMap tmap_out, Args A) {
  using C = Cfg<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Lay& L = A.L;
  const int cst = L.cst;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* cfull = bars;
  uint64_t* cfree = cfull + kMaxCStages;
  uint64_t* tfull = cfree + kMaxCStages;
  uint64_t* tfree = tfull + TSTAGES;
  uint64_t* a_ready = tfree + TSTAGES;
  uint64_t* a_free = a_ready + ASLOTS;
  uint64_t* acc_full = a_free + ASLOTS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* sh_full = acc_empty + 2;
  uint64_t* sh_empty = sh_full + 2;
  float* sh = reinterpret_cast<float*>(smem + L.sh);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.tmem_slot + 8);
  int* table = reinterpret_cast<int*>(smem + L.table);
  int* offs = table + (A.E + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile table: table[e] = first tile of expert e, table[E] = total (0 if offsets are invalid)
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
        cnt = o1 > o0 ? static_cast<int>((o1 - o0 + NMAX - 1) / NMAX) * A.n_tiles : 0;
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
    for (int s = 0; s < cst; ++s) {
      mbar_init(&cfull[s], 1);       // expect_tx by the code producer
      mbar_init(&cfree[s], 8);       // the dequant warps have read the codes
    }
    for (int s = 0; s < TSTAGES; ++s) {
      mbar_init(&tfull[s], 1);       // expect_tx by the token producer
      mbar_init(&tfree[s], C::kIssuers);   // tcgen05.commit of each issuer: tokens read
    }
    for (int a = 0; a < ASLOTS; ++a) {
      mbar_init(&a_ready[a], 8);     // the dequant warps' TMEM stores are complete
      mbar_init(&a_free[a], C::kIssuers);  // tcgen05.commit of each issuer: slot read
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], C::kIssuers);
      mbar_init(&acc_empty[b], C::kEpiWarps);
      mbar_init(&sh_full[b], 4);     // the dequant warps of the first k half
      mbar_init(&sh_empty[b], C::kEpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(C::kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = table[A.E];
  const int nst = A.nst;

  auto fail = [&](int lane_id) {
    if (lane_id == 0) { set_status(A.dev_status, W4_ERR_TIMEOUT); *abort_flag = 1; }
  };

  if (warp == 0) {
    // ---------------------------- code producer ----------------------------
    int slot = 0;
    uint32_t ph = 0;
    bool lap0 = true, ok = true;
    int64_t issued = 0;                        // code stages issued (lane 0)
    for (int t = blockIdx.x; t < total && ok && !*abort_flag; t += gridDim.x) {
      if (lane == 0) {
        if (t == static_cast<int>(blockIdx.x)) prefetch_tmap(&tmap_codes);
        Tile T;
        decode_tile(A, table, offs, t, NMAX, T);
        const int32_t row_a = static_cast<int32_t>(wrow(A, T, 0));
        const int32_t row_b = static_cast<int32_t>(wrow(A, T, kBM / 2));
        for (int st = 0; st < nst; ++st) {
          if (!lap0 && !mbar_wait(&cfree[slot], ph)) { ok = false; break; }
          uint8_t* cdst = smem + L.code + slot * C::kCodeStage;
          mbar_arrive_expect_tx(&cfull[slot], C::kCodeStage);
          tma_load_2d(cdst, &tmap_codes, st * (KSK / 8), row_a, &cfull[slot]);
          tma_load_2d(cdst + (kBM / 2) * C::kCodePitch, &tmap_codes, st * (KSK / 8), row_b, &cfull[slot]);
          ++issued;
          if (++slot == cst) { slot = 0; if (!lap0) ph ^= 1u; lap0 = false; }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (!ok) fail(lane);
    // After an abort the consumers stop waiting on the stages in flight: wait (bounded) until the
    // copies of the last cst stages issued have landed, so none lands after the CTA has exited.
    // Stage i used slot i % cst and completes phase (i / cst) of that slot's full barrier.
    if (lane == 0 && *abort_flag)
      for (int64_t i = issued > cst ? issued - cst : 0; i < issued; ++i)
        mbar_wait(&cfull[i % cst], static_cast<uint32_t>((i / cst) & 1));
    __syncwarp();
  } else if (warp == 3) {
    // ---------------------------- token producer ----------------------------
    if (lane == 0) {
      prefetch_tmap(&tmap_tok);
      int slot = 0;
      uint32_t ph = 0;
      bool lap0 = true, ok = true;
      int64_t issued = 0;                      // token stages issued
      for (int t = blockIdx.x; t < total && ok && !*abort_flag; t += gridDim.x) {
        Tile T;
        decode_tile(A, table, offs, t, NMAX, T);
        const int32_t r0 = static_cast<int32_t>(T.r0);
        for (int st = 0; st < nst; ++st) {
          if (!lap0 && !mbar_wait(&tfree[slot], ph)) { ok = false; break; }
          uint8_t* tdst = smem + C::tok + slot * C::kTokStage;
          mbar_arrive_expect_tx(&tfull[slot], C::kTokStage);
#pragma unroll
          for (int sub = 0; sub < C::kSubs; ++sub)
            tma_load_2d(tdst + sub * C::kTokSub, &tmap_tok, st * KSK + 64 * sub, r0, &tfull[slot]);
          ++issued;
          if (++slot == TSTAGES) { slot = 0; if (!lap0) ph ^= 1u; lap0 = false; }
        }
      }
      if (!ok) fail(0);
      if (*abort_flag)                         // (as for the code stages above)
        for (int64_t i = issued > TSTAGES ? issued - TSTAGES : 0; i < issued; ++i)
          mbar_wait(&tfull[i % TSTAGES], static_cast<uint32_t>((i / TSTAGES) & 1));
    }
    __syncwarp();
  } else if (warp == 1 || (warp >= C::kIssuerWarp0 && warp < C::kEpiWarp1)) {
    // ------------------------------ MMA issuers ------------------------------
    // One thread issues tcgen05.mma at about one instruction per 86+ cycles; C::kIssuers threads
    // (lane 0 of warp 1 and of warps 16, 17, ...) share each A slot: issuer i takes the token
    // columns [ns * NS, ns * NS + NS) (ns = i % NSPLIT) and the k16 blocks j with
    // j % KSPLIT == i / NSPLIT, accumulating into accumulator i / NSPLIT.
    const int iss = warp == 1 ? 0 : warp - 15;
    if (lane == 0 && iss < C::kIssuers) {
      const int nsi = iss % NSPLIT, ksi = iss / NSPLIT;
      int slot = 0, aslot = 0;
      uint32_t ph = 0, aph = 0;
      int ti = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
        Tile T;
        decode_tile(A, table, offs, t, NMAX, T);
        const int ab = ti % ABUF, use = ti / ABUF;
        if (ti >= ABUF && !mbar_wait(&acc_empty[ab], (use - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        int n_my = ((T.mrows + 15) & ~15) - nsi * C::kNS;       // this issuer's token columns
        n_my = n_my < 0 ? 0 : (n_my > C::kNS ? C::kNS : n_my);
        const uint32_t idesc = idesc_f16(kBM, n_my > 0 ? n_my : 16);
        const uint32_t d_tmem = tmem_base + C::acc_col(ab, ksi) + nsi * C::kNS;
        bool first = true;
        for (int st = 0; st < nst && ok; ++st) {
          if (!mbar_wait(&tfull[slot], ph)) { ok = false; break; }
          const uint32_t tb = smem_u32(smem + C::tok + slot * C::kTokStage) + nsi * C::kNS * 128;
          for (int hf = 0; hf < C::kHalves; ++hf) {
            if (!mbar_wait(&a_ready[aslot], aph)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_tm = tmem_base + C::kA0 + aslot * kACols;
            const int kleft = A.K - st * KSK - hf * 128;       // k of this slot inside K
            const int nk16 = kleft >= 128 ? 8 : (kleft > 0 ? kleft / 16 : 0);
            if (n_my > 0) {
              for (int j = ksi; j < nk16; j += KSPLIT) {
                const int jj = hf * 8 + j;                      // k16 block within the stage
                mma_f16_ts(d_tmem, a_tm + 8 * j,
                           sw128_desc(tb + (jj >> 2) * C::kTokSub + (jj & 3) * 32), idesc,
                           first ? 0u : 1u);
                first = false;
              }
            }
            mma_commit(&a_free[aslot]);    // the TMEM slot is free once these MMAs have read it
            if (++aslot == ASLOTS) { aslot = 0; aph ^= 1u; }
          }
          if (!ok) break;
          mma_commit(&tfree[slot]);        // and the token stage
          if (++slot == TSTAGES) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);         // accumulator ready once every MMA of the tile is done
      }
      if (!ok) fail(0);
    }
    __syncwarp();
  } else if ((warp >= 4 && warp < 8) || warp >= C::kEpiWarp1) {
    // ------------------------------ epilogue ------------------------------
    // TMEM lanes 32q .. 32q+31 are readable by warps with warp % 4 == q; with two epilogue warps
    // per quadrant, part cp takes the 16-column chunks cp, cp + 2, ...
    const int q = warp & 3;
    const int cp = warp < 8 ? 0 : 1;
    const int l = q * 32 + lane;
    const bool gelu = A.epi == W4_EPI_GELU_GATE;
    // A whole 16-token chunk is written to one of this warp's two 1 KB buffers as a [16 token]
    // x [32 outputs] (GELU: [16] x [16]) bf16 box and leaves by one TMA store, so the stores do
    // not hold the warp; a ragged chunk (the last of an expert's block) is stored element by
    // element and never touches the next block's rows.
    uint8_t* stg = smem + L.stage + (q + 4 * cp) * 2048;
    int n_out = 0;                                 // TMA stores issued by this warp (lane 0)
    int ti = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++ti) {
      Tile T;
      decode_tile(A, table, offs, t, NMAX, T);
      const int ab = ti % ABUF, hb = ti & 1;
      // the multipliers of the tile's tokens this warp finishes, loaded before the accumulator
      // wait so that their latency overlaps the tile's MMAs: with one warp per quadrant, lane l of
      // register m holds token 32m + l; with two, part cp finishes tokens 32j + 16cp + i (i < 16)
      // and lane l of register m holds the one with j = 2m + l / 16, i = l % 16
      constexpr int kRJ = NMAX / 32;
      constexpr int kRR = EPIW == 2 ? (kRJ + 1) / 2 : kRJ;
      float rmr[kRR];
#pragma unroll
      for (int m = 0; m < kRR; ++m) {
        const int tk = EPIW == 2 ? 32 * (2 * m + (lane >> 4)) + 16 * cp + (lane & 15) : 32 * m + lane;
        rmr[m] = tk < T.mrows ? __ldg(A.rowmul + T.r0 + tk) : 0.f;
      }
      if (!mbar_wait(&acc_full[ab], (ti / ABUF) & 1)) { fail(lane); break; }
      tc_fence_after();
      if (!mbar_wait(&sh_full[hb], (ti >> 1) & 1)) { fail(lane); break; }
      const float cm = sh[hb * kBM + l];          // 2^-e of this lane's weight row
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh_empty[hb]);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const int n_cols = (T.mrows + 15) & ~15;
      for (int c0 = 16 * cp; c0 < n_cols; c0 += 16 * EPIW) {
        // this chunk's multipliers: register c0 / 64 (two warps per quadrant) or c0 / 32 (one),
        // lanes sl .. sl + 15, picked by selects so that the array stays in registers
        const int m = EPIW == 2 ? c0 >> 6 : c0 >> 5;
        float rj = rmr[0];
#pragma unroll
        for (int mm = 1; mm < kRR; ++mm) rj = mm == m ? rmr[mm] : rj;
        const int sl = EPIW == 2 ? (c0 & 32) >> 1 : c0 & 16;
        float v[16];
        tmem_ld16(taddr + C::acc_col(ab, 0) + c0, v);
#pragma unroll
        for (int kp = 1; kp < KSPLIT; ++kp) {        // the issuers' k parts, summed in order
          float w[16];
          tmem_ld16(taddr + C::acc_col(ab, kp) + c0, w);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += w[i];
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (v[i] * __shfl_sync(0xffffffffu, rj, sl + i)) * cm;
        if (A.tma_out && c0 + 16 <= T.mrows) {
          uint16_t* buf = reinterpret_cast<uint16_t*>(stg + (n_out & 1) * 1024);
          if (n_out >= 2) {                         // the store that last read this buffer
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          if (gelu) {
            const bool upper = lane >= 16;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float send = upper ? v[i] : v[8 + i];
              const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
              const float g = upper ? recv : v[i];
              const float u = upper ? v[8 + i] : recv;
              buf[(i + (upper ? 8 : 0)) * 16 + (lane & 15)] = f32_to_bf16_bits(gelu_tanh(g) * u);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) buf[i * 32 + lane] = f32_to_bf16_bits(v[i]);
          }
          fence_proxy_async();                      // the generic writes, before the async read
          __syncwarp();
          if (lane == 0) {
            const int x = gelu ? T.nt * (kBM / 2) + 16 * q : T.nt * kBM + 32 * q;
            tma_store_2d(&tmap_out, x, static_cast<int32_t>(T.r0 + c0), buf);
            bulk_commit();
          }
          ++n_out;
        } else if (gelu) {
          // lanes i < 16: gate values, lanes i + 16: up values of the same output j; the lower
          // lane finishes tokens c0 .. c0+7, the upper one tokens c0+8 .. c0+15
          const bool upper = lane >= 16;
          const int Nh = A.N >> 1;
          const int j = T.nt * (kBM / 2) + 16 * q + (lane & 15);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float send = upper ? v[i] : v[8 + i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const float g = upper ? recv : v[i];
            const float u = upper ? v[8 + i] : recv;
            const int tk = c0 + i + (upper ? 8 : 0);
            if (tk < T.mrows)
              A.out[(T.r0 + tk) * Nh + j] = f32_to_bf16_bits(gelu_tanh(g) * u);
          }
        } else {
          const int n = T.nt * kBM + l;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int tk = c0 + i;
            if (tk < T.mrows) A.out[(T.r0 + tk) * A.N + n] = f32_to_bf16_bits(v[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
    if (lane == 0) bulk_wait_all();              // this warp's stores are complete before exit
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------ dequant ------------------------------
    // warp 8 + 4h + q: TMEM lanes 32q .. 32q+31 (one weight row each), and in every 128-k slot the
    // groups 2h and 2h + 1 (TMEM columns 32h .. 32h + 31 of the slot)
    const int dw = warp - 8;
    const int q = dw & 3, h = dw >> 2;
    const int l = q * 32 + lane;
    const int r = lane_row(A.epi, l);
    // swizzle phase of code row r: 64-byte swizzle XORs the 16-byte chunk with address bits 7-8
    // ((r >> 1) & 3 at a 64-byte pitch), 128-byte swizzle with bits 7-9 (r & 7 at a 128-byte pitch)
    const int sw = KSK == 128 ? ((r >> 1) & 3) : (r & 7);
    const uint32_t tlane = static_cast<uint32_t>(q * 32) << 16;
    // Scale queue: the word holding groups g0, g0 + 1 of this row for each (tile, stage, half) in
    // order, kSQ entries ahead of the dequantisation, loaded from global memory (L2-resident
    // after the first touch of a 32-byte sector), across tile boundaries.
    constexpr int kSQ = 3;
    uint32_t sq[kSQ];
    int pf_t = blockIdx.x, pf_st = 0, pf_hf = 0;
    const uint32_t* pf_row = nullptr;            // this thread's scale row in tile pf_t
    auto pf_tile = [&]() {
      if (pf_t < total) {
        Tile P;
        decode_tile(A, table, offs, pf_t, NMAX, P);
        pf_row = reinterpret_cast<const uint32_t*>(A.scales + wrow(A, P, r) * A.kg);
      }
    };
    auto pf_next = [&]() -> uint32_t {
      uint32_t v = 0u;
      if (pf_t < total) {
        const int g0 = pf_st * (KSK / 32) + 4 * pf_hf + 2 * h;
        if (g0 < A.kg) v = __ldg(pf_row + (g0 >> 1));     // groups past K: scale 0
        if (++pf_hf == C::kHalves) {
          pf_hf = 0;
          if (++pf_st == nst) { pf_st = 0; pf_t += gridDim.x; pf_tile(); }
        }
      }
      return v;
    };
    pf_tile();
#pragma unroll
    for (int i = 0; i < kSQ; ++i) sq[i] = pf_next();
    // exponent of this row, one tile ahead
    int e_next = 0;
    if (blockIdx.x < static_cast<unsigned>(total)) {
      Tile T0;
      decode_tile(A, table, offs, blockIdx.x, NMAX, T0);
      e_next = A.rowexp[wrow(A, T0, r)];
    }
    int slot = 0, aslot = 0;
    uint32_t ph = 0, aph = 0;
    bool alap0 = true;
    int ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
      const int sb = ti & 1;
      const int e = e_next;
      if (t + static_cast<int>(gridDim.x) < total) {
        Tile Tn;
        decode_tile(A, table, offs, t + gridDim.x, NMAX, Tn);
        e_next = A.rowexp[wrow(A, Tn, r)];
      }
      // e brings the row's largest finite |scale| to [2^10, 2^11), so 24 s' stays below 2^16 and
      // every scale within 2^21 of the largest keeps s'' and 24 s' exact
      const float smul = pow2f(e - 6);
      if (h == 0) {
        if (ti >= 2 && !mbar_wait(&sh_empty[sb], ((ti >> 1) - 1) & 1)) { ok = false; break; }
        sh[sb * kBM + l] = pow2f(-e);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh_full[sb]);
      }
      for (int st = 0; st < nst; ++st) {
        if (!mbar_wait(&cfull[slot], ph)) { ok = false; break; }
        const uint32_t cbase = smem_u32(smem + L.code + slot * C::kCodeStage) + r * C::kCodePitch;
        // this thread's groups: 4 hf + 2h and 4 hf + 2h + 1 of each 128-k half hf of the stage
        uint4 wv[2 * C::kHalves];
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
#pragma unroll
          for (int i = 0; i < 2; ++i) wv[2 * hf + i] = lds128(cbase + (((4 * hf + 2 * h + i) ^ sw) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&cfree[slot]);
        if (++slot == cst) { slot = 0; ph ^= 1u; }
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf) {
          const uint32_t sv = sq[0];
#pragma unroll
          for (int i = 0; i + 1 < kSQ; ++i) sq[i] = sq[i + 1];
          sq[kSQ - 1] = pf_next();
          uint32_t s2a, c2a, s2b, c2b;
          scale_pair(sv & 0xFFFFu, smul, s2a, c2a);
          scale_pair(sv >> 16, smul, s2b, c2b);
          const uint4 w0 = wv[2 * hf], w1 = wv[2 * hf + 1];
          uint32_t o[32];
          deq_word(w0.x, s2a, c2a, o + 0);
          deq_word(w0.y, s2a, c2a, o + 4);
          deq_word(w0.z, s2a, c2a, o + 8);
          deq_word(w0.w, s2a, c2a, o + 12);
          deq_word(w1.x, s2b, c2b, o + 16);
          deq_word(w1.y, s2b, c2b, o + 20);
          deq_word(w1.z, s2b, c2b, o + 24);
          deq_word(w1.w, s2b, c2b, o + 28);
          if (!alap0 && !mbar_wait(&a_free[aslot], aph ^ 1u)) { ok = false; break; }
          tc_fence_after();
          tmem_st32(tmem_base + tlane + C::kA0 + aslot * kACols + 32 * h, o);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_ready[aslot]);
          if (++aslot == ASLOTS) { aslot = 0; aph ^= 1u; alap0 = false; }
        }
        if (!ok) break;
      }
      if (!ok) break;
    }
    if (!ok) fail(lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols) : "memory");
  }
}

}  // namespace tm
}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 tm_encode_fn() {
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

bool w4_tm_supported(int N, int K, int epi) {
  const int kg = K / 32;
  if (K % 64 || kg > w4::tm::kMaxKg) return false;
  if (epi == W4_EPI_GELU_GATE) return (N / 2) % (w4::tm::kBM / 2) == 0;
  return N % w4::tm::kBM == 0;
}

// shared memory of one CTA (the opt-in maximum minus the 1024-byte alignment slack)
constexpr int kTmSmemBudget = 232448 - 1024;

template <int NMAX, int KSK, int TSTAGES, int ASLOTS, int NSPLIT, int KSPLIT, int ABUF, int EPIW>
static bool tm_layout(int E, int kg, w4::tm::Lay& L) {
  using C = w4::tm::Cfg<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>;
  (void)kg;
  L.code = C::code;
  const int stage = C::kEpiWarps * 2048;
  const int fixed = stage + 2 * w4::tm::kBM * 4 + C::nbars * 8 + 16 + (E + 1) * 8;
  int cst = (kTmSmemBudget - L.code - fixed) / C::kCodeStage;
  if (cst > w4::tm::kMaxCStages) cst = w4::tm::kMaxCStages;
  if (cst < 2) return false;
  L.cst = cst;
  L.stage = L.code + cst * C::kCodeStage;     // 1024-byte aligned (whole code stages)
  L.sh = L.stage + stage;
  L.bars = L.sh + 2 * w4::tm::kBM * 4;
  L.tmem_slot = L.bars + C::nbars * 8;
  L.table = L.tmem_slot + 16;
  L.total = L.table + (E + 1) * 8;
  return L.total <= kTmSmemBudget;
}

template <int NMAX, int KSK, int TSTAGES, int ASLOTS, int NSPLIT, int KSPLIT, int ABUF, int EPIW>
static w4_status tm_launch_cfg(const uint32_t* codes, const uint16_t* a16, int64_t rows, int K,
                               w4::tm::Args A, cudaStream_t stream, int sm_count) {
  using C = w4::tm::Cfg<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>;
  auto fn = tm_encode_fn();
  if (!fn) return W4_ERR_CUDA;
  if (!tm_layout<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>(A.E, A.kg, A.L)) return W4_ERR_UNSUPPORTED;
  A.nst = (K + KSK - 1) / KSK;
  cuuint32_t estr[2] = {1, 1};
  // raw codes [E*N, K/8] words: box = one stage of k (KSK/8 words) x 64 rows, swizzled to the
  // row pitch (64 bytes: 64-byte swizzle, 128 bytes: 128-byte swizzle)
  CUtensorMap tmap_codes;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 8), static_cast<cuuint64_t>(A.E) * A.N};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 8) * 4};
    cuuint32_t box[2] = {KSK / 8, static_cast<cuuint32_t>(w4::tm::kBM / 2)};
    if (fn(&tmap_codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           KSK == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return W4_ERR_CUDA;
  }
  // converted token rows [rows, K] fp16: box = 64 k x NMAX rows, 128-byte swizzle
  CUtensorMap tmap_tok;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(NMAX)};
    if (fn(&tmap_tok, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(a16), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return W4_ERR_CUDA;
  }
  // routed outputs [rows, N] (GELU: [rows, N / 2]) bf16: box = 32 (GELU: 16) outputs x 16 rows,
  // unswizzled, for the epilogue's whole-chunk stores; without a usable map every element is
  // stored directly
  CUtensorMap tmap_out;
  std::memset(&tmap_out, 0, sizeof(tmap_out));
  A.tma_out = 0;
  {
    const bool gelu = A.epi == W4_EPI_GELU_GATE;
    const int64_t nout = gelu ? A.N / 2 : A.N;
    if ((reinterpret_cast<uintptr_t>(A.out) & 15) == 0 && (nout * 2) % 16 == 0 && rows >= 16) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(nout), static_cast<cuuint64_t>(rows)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(nout) * 2};
      cuuint32_t box[2] = {gelu ? 16u : 32u, 16u};
      if (fn(&tmap_out, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, A.out, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
        A.tma_out = 1;
    }
  }
  const size_t smem = static_cast<size_t>(A.L.total) + 1024;
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::tm::tm_gemm_kernel<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 232448) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  w4::tm::tm_gemm_kernel<NMAX, KSK, TSTAGES, ASLOTS, NSPLIT, KSPLIT, ABUF, EPIW>
      <<<sm_count, 32 * C::kWarps, smem, stream>>>(tmap_codes, tmap_tok, tmap_out, A);
  return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_launch_tm_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                            const uint32_t* codes, const uint16_t* scales, const int32_t* offsets,
                            int E, int64_t rows, int N, int K, int epi, uint16_t* out, void* ws,
                            size_t ws_bytes, int32_t* dev_status, cudaStream_t stream, int sm_count) {
  if (!w4_tm_supported(N, K, epi)) return W4_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(scales) & 3) != 0) return W4_ERR_UNSUPPORTED;
  if (rows == 0) return W4_OK;
  if (rows >= (1LL << 31) || static_cast<int64_t>(E) * N >= (1LL << 31)) return W4_ERR_UNSUPPORTED;
  const int kd = k_div > 0 ? k_div : 1;
  const int64_t a_rows = a_row_of_pair ? rows / kd : rows;   // rows of `a` a pair may name
  if (a_rows <= 0) return W4_ERR_INVALID_ARG;
  const int64_t wrows = static_cast<int64_t>(E) * N;
  if (!ws || ws_bytes < w4_tc_workspace_bytes(rows, K, wrows) || (reinterpret_cast<uintptr_t>(ws) & 15))
    return W4_ERR_WORKSPACE;
  w4_launch_a_to_f16(a, a_row_of_pair, kd, a_rows, rows, K, scales, wrows, ws, dev_status, stream,
                     sm_count);

  w4::tm::Args A{};
  A.rowmul = w4_ws_rowmul(ws, rows, K);
  A.rowexp = w4_ws_rowexp(ws, rows, K);
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32;
  A.rows = rows; A.epi = epi; A.out = out;
  A.n_tiles = (epi == W4_EPI_GELU_GATE) ? (N / 2) / (w4::tm::kBM / 2) : N / w4::tm::kBM;
  A.dev_status = dev_status;
  const uint16_t* a16 = w4_ws_a16(ws);
  // 192-row token blocks, 128-k stages with three token stages in flight, one MMA-issuing thread
  // (N = 192: every tcgen05.mma costs a fixed time on top of its columns, so fewer, wider MMAs
  // finish sooner than two threads' 96-column ones), two 192-column accumulators drained by eight
  // epilogue warps
  return tm_launch_cfg<192, 128, 3, 2, 1, 1, 2, 2>(codes, a16, rows, K, A, stream, sm_count);
}
