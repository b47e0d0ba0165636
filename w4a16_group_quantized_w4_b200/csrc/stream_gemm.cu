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
#include <cstring>

#include "stream_gemm.cuh"

namespace w4 {
template <int MT, int GS, bool GELU, int SCALE, bool ZP, int SPL>
__global__ void __launch_bounds__(kThreads, 1)
stream_gemm_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, const __grid_constant__ StreamArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  stream_gemm_body<MT, GS, GELU, SCALE, ZP, SPL>(tmap_codes, tmap_scales, A, smem_raw);
}

template <int MT, int GS, bool ZP, bool CHUNK>
__global__ void __launch_bounds__(256)
stream_prep_kernel(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair, int k_div,
                   int64_t a_rows, int64_t rows, int K, const int32_t* __restrict__ offsets, int E,
                   uint8_t* __restrict__ xw, int n_stages, int64_t n_blocks, int32_t* __restrict__ counters,
                   int n_counters, int32_t* dev_status, int bchunk) {
  extern __shared__ int prep_smem[];
  // The GEMM after this pass may launch only once the kernels before the pass have completed
  // (it reads the routing and starts its weight stream before waiting for this pass).
  pdl_wait();
  pdl_trigger();
  stream_prep_body<MT, GS, ZP, false, CHUNK>(a, a_row_of_pair, k_div, a_rows, rows, K, offsets, E, xw, n_stages,
                                             n_blocks, counters, n_counters, dev_status, prep_smem, bchunk);
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
static w4::Layout make_layout(int MT, int GS, int scale_mode, int kg, int E, bool zp) {
  w4::Layout L{};
  L.sc_bytes = scale_mode == w4::kScaleTma ? 2 * w4::kHalf * GS * 2
             : scale_mode == w4::kScaleBlock ? 2 * w4::kHalf * kg * 2 : 0;
  L.slot_bytes = (w4::slot_sc_off(MT, GS, zp) + L.sc_bytes + 1023) & ~1023;
  const int table_bytes = (E + 1) * 12;
  const int red_bytes = 2 * 4 * (MT / 8) * 2 * 32 * 16;
  const int budget = ((w4::kSmemPerCta - 1024 - table_bytes) / w4::kPipes) & ~1023;   // per pipeline
  const int fixed = red_bytes + (2 * w4::kMaxStages + 1) * 8 + 16 + 128;
  int S = (budget - fixed) / L.slot_bytes;
  if (S > w4::kMaxStages) S = w4::kMaxStages;
  L.stages = S;
  int off = S * L.slot_bytes;
  L.red_off = off;                               // (16-byte aligned: slots are 1 KB)
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

template <int MT, int GS, bool GELU, int SCALE, bool ZP, int SPL>
static w4_status launch_one(const CUtensorMap& tmap, const CUtensorMap& smap, const w4::StreamArgs& A,
                            int sm_count, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(w4::stream_gemm_kernel<MT, GS, GELU, SCALE, ZP, SPL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, w4::kSmemPerCta) != cudaSuccess)
      return W4_ERR_CUDA;
    attr_done[dev] = 1;
  }
  return launch_pdl(w4::stream_gemm_kernel<MT, GS, GELU, SCALE, ZP, SPL>, dim3(sm_count), dim3(w4::kThreads),
                    A.L.total, stream, tmap, smap, A) == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

template <int MT, int GS, bool GELU, int SCALE, bool ZP>
static w4_status launch_split(const CUtensorMap& tmap, const CUtensorMap& smap, const w4::StreamArgs& A,
                              int sm_count, cudaStream_t stream) {
  return A.splits > 1 ? launch_one<MT, GS, GELU, SCALE, ZP, 1>(tmap, smap, A, sm_count, stream)
                      : launch_one<MT, GS, GELU, SCALE, ZP, 0>(tmap, smap, A, sm_count, stream);
}

template <int MT, int GS, bool GELU>
static w4_status launch_scale(int scale_mode, bool zp, const CUtensorMap& tmap, const CUtensorMap& smap,
                              const w4::StreamArgs& A, int sm_count, cudaStream_t stream) {
  if (zp) return launch_split<MT, GS, GELU, w4::kScaleLdg, true>(tmap, smap, A, sm_count, stream);
  if (scale_mode == w4::kScaleTma) return launch_split<MT, GS, GELU, w4::kScaleTma, false>(tmap, smap, A, sm_count, stream);
  if (scale_mode == w4::kScaleBlock) return launch_split<MT, GS, GELU, w4::kScaleBlock, false>(tmap, smap, A, sm_count, stream);
  return launch_split<MT, GS, GELU, w4::kScaleLdg, false>(tmap, smap, A, sm_count, stream);
}

template <int MT, int GS, bool ZP>
static cudaError_t launch_prep_z(dim3 grid, size_t smem, cudaStream_t stream, const uint16_t* a,
                                 const int32_t* a_row_of_pair, int kd, int64_t a_rows, int64_t rows, int K,
                                 const int32_t* offsets, int E, uint8_t* xw, int n_stages, int64_t n_blocks,
                                 int32_t* counters, int n_counters, int32_t* dev_status, int bchunk, bool chunk) {
  if (chunk)
    return launch_pdl(w4::stream_prep_kernel<MT, GS, ZP, true>, grid, dim3(256), smem, stream, a, a_row_of_pair, kd,
                      a_rows, rows, K, offsets, E, xw, n_stages, n_blocks, counters, n_counters, dev_status, bchunk);
  return launch_pdl(w4::stream_prep_kernel<MT, GS, ZP, false>, grid, dim3(256), smem, stream, a, a_row_of_pair, kd,
                    a_rows, rows, K, offsets, E, xw, n_stages, n_blocks, counters, n_counters, dev_status, bchunk);
}

template <int MT, int GS>
static cudaError_t launch_prep(bool zp, dim3 grid, size_t smem, cudaStream_t stream, const uint16_t* a,
                               const int32_t* a_row_of_pair, int kd, int64_t a_rows, int64_t rows, int K,
                               const int32_t* offsets, int E, uint8_t* xw, int n_stages, int64_t n_blocks,
                               int32_t* counters, int n_counters, int32_t* dev_status, int bchunk, bool chunk) {
  if (zp)
    return launch_prep_z<MT, GS, true>(grid, smem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offsets, E, xw,
                                       n_stages, n_blocks, counters, n_counters, dev_status, bchunk, chunk);
  return launch_prep_z<MT, GS, false>(grid, smem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offsets, E, xw,
                                      n_stages, n_blocks, counters, n_counters, dev_status, bchunk, chunk);
}

w4_status w4_stream_setup(const uint32_t* codes, const uint16_t* scales, const int32_t* offsets, int E,
                          int64_t rows, int N, int K, int epi, int32_t* dev_status, int sm_count,
                          uint64_t wait_ns, int stall_after, const uint8_t* zeros, int group, StreamCall& C,
                          bool allow_block) {
  const bool dense = (offsets == nullptr);
  const bool zp = zeros != nullptr;
  int gshift = 0;
  while ((32 << gshift) < group) ++gshift;
  if ((32 << gshift) != group || K % group) return W4_ERR_INVALID_ARG;   // (callers check first)
  StreamPlan p = plan_stream(rows, N, K, E, epi, dense, sm_count);
  w4::StreamArgs A{};
  A.scales = scales; A.offsets = offsets;
  A.E = E; A.N = N; A.K = K; A.kg = K / 32; A.rows = rows; A.epi = epi;
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
  } else if (allow_block && A.kg % 2 == 0 && A.kg <= w4::kBlockMaxKg && N % 8 == 0 && s16 &&
             (epi == W4_EPI_GELU_GATE ? (N / 2) % w4::kHalf == 0 : N % w4::kBN == 0)) {
    // (whole tiles only: the 64-row blocks are plain bulk copies and must stay inside the array)
    scale_mode = w4::kScaleBlock;
  } else {
    scale_mode = w4::kScaleLdg;
  }
  A.L = make_layout(p.MT, p.GS, scale_mode, A.kg, E, zp);
  if (A.L.stages < 2) return W4_ERR_UNSUPPORTED;
  C.A = A;
  C.p = p;
  C.scale_mode = scale_mode;
  C.n_blocks = block_capacity(rows, p.MT, E, dense);
  C.prep_bytes = prep_bytes(p, rows, E, dense, zp);
  C.counters_bytes = p.splits > 1 ? counters_bytes(p, rows, E, dense) : 0;
  C.partial_bytes = p.splits > 1 ? static_cast<size_t>(p.splits) * rows * N * sizeof(float) : 0;
  std::memset(&C.smap, 0, sizeof(C.smap));
  std::memset(&C.tmap, 0, sizeof(C.tmap));
  if (rows == 0) return W4_OK;
  if (!encode_codes_map(&C.tmap, codes, static_cast<int64_t>(E) * N, K)) return W4_ERR_CUDA;
  if (scale_mode == w4::kScaleTma &&
      !encode_scales_map(&C.smap, scales, static_cast<int64_t>(E) * N, A.kg, p.GS))
    return W4_ERR_CUDA;
  return W4_OK;
}

void w4_stream_bind(StreamCall& C, uint8_t* ws) {
  C.A.xw = ws;
  if (C.p.splits > 1) {
    C.A.counters = reinterpret_cast<int32_t*>(ws + C.prep_bytes);
    C.A.partial = reinterpret_cast<float*>(ws + C.prep_bytes + C.counters_bytes);
  }
}

w4_status w4_launch_stream_gemm(const uint16_t* a, const int32_t* a_row_of_pair, int k_div,
                                const uint32_t* codes, const uint16_t* scales,
                                const int32_t* offsets, int E, int64_t rows, int N, int K, int epi,
                                uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                                cudaStream_t stream, int sm_count, uint64_t wait_ns, int stall_after,
                                const uint8_t* zeros, int group) {
  const bool dense = (offsets == nullptr);
  const bool zp = zeros != nullptr;
  StreamCall C;
  const w4_status st = w4_stream_setup(codes, scales, offsets, E, rows, N, K, epi, dev_status, sm_count, wait_ns,
                                       stall_after, zeros, group, C);
  if (st != W4_OK || rows == 0) return st;
  const size_t need = w4_stream_workspace_bytes(rows, N, K, E, epi, dense, sm_count, zp);
  if (ws == nullptr || ws_bytes < need) return W4_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  w4_stream_bind(C, wsb);
  C.A.out = out;
  const StreamPlan& p = C.p;
  {
    // (the preparation pass clears the split-K arrival counters)
    const int kd = k_div > 0 ? k_div : 1;
    const int64_t a_rows = a_row_of_pair ? rows / kd : rows;
    // A few rows (GEMVs, one-token decode) are cut into pieces of bchunk 256-k blocks, one warp
    // each (every piece finds the row's exponent itself), so that about 256 warps share the
    // conversion instead of one warp per row working through it alone.
    const int nblk = p.n_stages * (p.GS / w4::kBoxG);
    const int64_t want = rows >= 256 ? 1 : std::min<int64_t>(nblk, 256 / rows);
    const int bchunk = static_cast<int>((nblk + want - 1) / want);
    const int64_t items = rows * ((nblk + bchunk - 1) / bchunk);
    const int64_t wblocks = (items + 7) / 8;
    const int grid = static_cast<int>(wblocks < 16LL * sm_count ? wblocks : 16LL * sm_count);
    const int n_counters = static_cast<int>(C.counters_bytes / sizeof(int32_t));
    const size_t psmem = dense ? 0 : static_cast<size_t>(E + 1) * 2 * sizeof(int);
    const int32_t* offs = dense ? nullptr : offsets;
    const cudaError_t e = p.MT == 8
        ? launch_prep<8, 16>(zp, dim3(grid), psmem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offs, E, wsb,
                             p.n_stages, C.n_blocks, C.A.counters, n_counters, dev_status, bchunk, bchunk < nblk)
        : launch_prep<16, 8>(zp, dim3(grid), psmem, stream, a, a_row_of_pair, kd, a_rows, rows, K, offs, E, wsb,
                             p.n_stages, C.n_blocks, C.A.counters, n_counters, dev_status, bchunk, bchunk < nblk);
    if (e != cudaSuccess) return W4_ERR_CUDA;
  }
  const bool gelu = epi == W4_EPI_GELU_GATE;
  const w4::StreamArgs& A = C.A;
  if (p.MT == 8)
    return gelu ? launch_scale<8, 16, true>(C.scale_mode, zp, C.tmap, C.smap, A, sm_count, stream)
                : launch_scale<8, 16, false>(C.scale_mode, zp, C.tmap, C.smap, A, sm_count, stream);
  return gelu ? launch_scale<16, 8, true>(C.scale_mode, zp, C.tmap, C.smap, A, sm_count, stream)
              : launch_scale<16, 8, false>(C.scale_mode, zp, C.tmap, C.smap, A, sm_count, stream);
}
