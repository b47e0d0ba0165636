// Fused MoE decode layer: routing, the gate/up grouped GEMM with the GELU gate, the down grouped
// GEMM and the combine in ONE persistent kernel launch.
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "What changed in vLLM's TPU backend": the fused-MoE layer routes every token to its top-k
// experts and runs the experts' packed int4 weights through one grouped matmul with per-group
// scales; section "The gap at 26B" gives the shape (128 experts, 8 active).  The layer computes
// exactly what moe_route_permute, moe_w4a16_gmm (gate/up, GELU gate), moe_w4a16_gmm (down) and
// moe_combine compute on the weight-streaming kernel, with the same arithmetic in the same order,
// so its y is bit-identical to theirs.
//
// Design (sm_100a, one CTA per SM, cooperative launch so that every CTA is resident).  The GEMM
// units go round robin from the first CTA, so serial work (routing, row preparation, combine) is
// handed out from the last CTA down, where the pipelines are idle at small batches.
//   1. routing: the top-k of each token on one warp (token t on CTA G-1-t), each adding one to a
//      counter; the last CTA then forms the expert offsets and the permutation from the top-k
//      and raises a flag that every CTA waits for.
//   2. gate/up GEMM (the weight-streaming kernel's body) with its records prepared in the same
//      phase: the producers start the weight stream at once while the compute warps first write
//      the routed rows' records (one warp per row), each adding one to its token block's ready
//      counter; a producer copies a block's records once that counter has reached the block's row
//      count.  Every finished (block, weight tile) adds one to the block's done counter after its
//      h outputs are written.
//   3. down GEMM, the same way on h: a row's records are prepared once its block's gate/up tiles
//      are all done, while the producers already stream the down weights.
//   4. combine: a warp per (token, 256 features) waits for the down tiles of the token's k rows
//      and forms y in slot order.
// No phase waits for the whole grid: each waits only for what it reads.  Every wait is bounded
// (W4_ERR_TIMEOUT).  The counters live in a control area at the front of the workspace; the
// last CTA to finish clears it, so each call starts from zero.
#include <algorithm>
#include <cstring>

#include "route.cuh"
#include "stream_gemm.cuh"

namespace w4 {

constexpr int kLayerMaxT = kFusedMaxT;        // tokens per call (single-CTA routing)
constexpr int kLayerCtlHeader = 64;           // ints: [0] routing written, [1] CTAs finished,
                                              // [2] tokens whose top-k is written

struct LayerArgs {
  RouteArgs R;              // logits, T, E, k and the routing outputs (workspace)
  const uint16_t* x;        // [T, H]
  StreamArgs gu, dn;        // gate/up (out = h [T k, I]) and down (out = o [T k, H])
  int32_t* ctl;             // control area (ctl_words ints, zero at entry, cleared at exit)
  int ctl_words;
  int32_t* ready_gu;        // [n_blocks] rows of the block whose gate/up records are written
  int32_t* done_gu;         // [n_blocks] gate/up tiles of the block whose h is written
  int32_t* ready_dn;        // [n_blocks] rows of the block whose down records are written
  int32_t* done_dn;         // [n_blocks] down tiles of the block whose o is written
  int32_t* row_blk;         // [T k] token block of each routed row
  int64_t n_blocks;
  uint16_t* y;              // [T, H]
  int H, I;
  int32_t* dev_status;
  uint64_t wait_ns;
};

// y[t] = sum_j w[t, j] * o[pair_pos[t k + j]], float32 in slot order (the order of
// combine_kernel), bf16 out.  One warp per (token, run of 32 chunks of 8 features); lanes
// 0..k-1 first wait for their row's down tiles.
__device__ __forceinline__ void layer_combine(const LayerArgs& P) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int T = P.R.T, k = P.R.k;
  const int nch = P.H >> 3;
  const int nrun = (nch + 31) >> 5;
  const int64_t Tk = static_cast<int64_t>(T) * k;
  const int64_t items = static_cast<int64_t>(T) * nrun;
  const int rb = gridDim.x - 1 - blockIdx.x;
  for (int64_t it = static_cast<int64_t>(threadIdx.x >> 5) * gridDim.x + rb; it < items;
       it += static_cast<int64_t>(gridDim.x) * wpb) {
    const int t = static_cast<int>(it / nrun);
    const int run = static_cast<int>(it - static_cast<int64_t>(t) * nrun);
    int pos = -1;
    float w = 0.f;
    if (lane < k) {
      pos = __ldcg(P.R.pair_pos + static_cast<int64_t>(t) * k + lane);
      w = __ldcg(P.R.topk_w + static_cast<int64_t>(t) * k + lane);
      if (pos < 0 || pos >= Tk) {
        pos = -1;                                       // not a valid permutation entry: skipped
      } else {
        const int b = __ldcg(P.row_blk + pos);
        if (b < 0 || b >= P.n_blocks) {
          set_status(P.dev_status, W4_ERR_INVALID_ARG);
          pos = -1;
        } else if (!wait_count(P.done_dn + b, P.dn.n_tiles, P.wait_ns)) {
          set_status(P.dev_status, W4_ERR_TIMEOUT);
        }
      }
    }
    __syncwarp();
    const int c = run * 32 + lane;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    // eight rows at a time: their loads in flight together, then the sums in slot order
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 v[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        v[jj] = make_uint4(0, 0, 0, 0);
        const int pj = __shfl_sync(0xffffffffu, pos, (j0 + jj) & 31);
        if (j0 + jj < k && pj >= 0 && c < nch)
          v[jj] = __ldcg(reinterpret_cast<const uint4*>(P.dn.out + static_cast<int64_t>(pj) * P.H) + c);
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const float wj = __shfl_sync(0xffffffffu, w, (j0 + jj) & 31);
        if (j0 + jj < k) {
          const uint32_t vv[4] = {v[jj].x, v[jj].y, v[jj].z, v[jj].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(wj, bf16_lo_to_f32(vv[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj, bf16_hi_to_f32(vv[i]), acc[2 * i + 1]);
          }
        }
      }
    }
    if (c < nch) {
      uint4 out;
      out.x = pack_bf16x2(acc[0], acc[1]);
      out.y = pack_bf16x2(acc[2], acc[3]);
      out.z = pack_bf16x2(acc[4], acc[5]);
      out.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(P.y + static_cast<int64_t>(t) * P.H)[c] = out;
    }
  }
}

template <int SGU, int SDN>
__global__ void __launch_bounds__(kThreads, 1)
moe_layer_kernel(const __grid_constant__ CUtensorMap gu_tmap, const __grid_constant__ CUtensorMap gu_smap,
                 const __grid_constant__ CUtensorMap dn_tmap, const __grid_constant__ CUtensorMap dn_smap,
                 const __grid_constant__ LayerArgs P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  int* smem_i = reinterpret_cast<int*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int rb = G - 1 - blockIdx.x;                 // rank from the last CTA
  const int64_t rows = static_cast<int64_t>(P.R.T) * P.R.k;

  // 1. routing: top-k per token, then offsets and permutation on the last CTA
  for (int t = warp * G + rb; t < P.R.T; t += G * (blockDim.x >> 5)) {
    route_topk_one(P.R, t);
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(P.ctl + 2, 1);
    }
  }
  if (rb == 0) {
    int ready = 1;
    if (tid == 0 && !wait_count(P.ctl + 2, P.R.T, P.wait_ns)) {
      ready = 0;
      set_status(P.dev_status, W4_ERR_TIMEOUT);
    }
    if (__syncthreads_and(ready)) route_fused_body<false, true>(P.R, smem_i);
    fence_proxy_async_smem();        // (this shared memory is next written by bulk copies)
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      atomicAdd(P.ctl, 1);
    }
  }
  int ok = 1;
  if (tid == 0 && !wait_count(P.ctl, 1, P.wait_ns)) {
    ok = 0;
    set_status(P.dev_status, W4_ERR_TIMEOUT);
  }
  ok = __syncthreads_and(ok);
  if (ok) {
    const int64_t ncw = static_cast<int64_t>(G) * (kPipes * kWarps);   // compute warps of the grid
    // 2. gate/up GEMM with the GELU gate -> h; its compute warps first prepare the routed rows
    const auto pre_gu = [&](const int* offs, const int* blk, int cw, int) {
      const PrepHooks h{nullptr, 0, P.ready_gu, P.row_blk, P.wait_ns};
      stream_prep_rows<8, 16, false, true>(P.x, P.R.sorted_pair, P.R.k, P.R.T, rows, P.H, true, offs, blk, P.R.E,
                                           const_cast<uint8_t*>(P.gu.xw), P.gu.n_stages, P.n_blocks, P.dev_status,
                                           h, static_cast<int64_t>(cw) * G + rb, ncw);
    };
    stream_gemm_body<8, 16, true, SGU, false, 2, true>(gu_tmap, gu_smap, P.gu, smem_raw, pre_gu);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) stream_gemm_inval(P.gu.L, smem_raw);
    __syncthreads();
    // 3. down GEMM -> o; its compute warps first prepare h's rows as their blocks complete
    const auto pre_dn = [&](const int* offs, const int* blk, int cw, int) {
      const PrepHooks h{P.done_gu, P.gu.n_tiles, P.ready_dn, nullptr, P.wait_ns};
      stream_prep_rows<8, 16, false, true>(P.gu.out, nullptr, 1, rows, rows, P.I, true, offs, blk, P.R.E,
                                           const_cast<uint8_t*>(P.dn.xw), P.dn.n_stages, P.n_blocks, P.dev_status,
                                           h, static_cast<int64_t>(cw) * G + rb, ncw);
    };
    stream_gemm_body<8, 16, false, SDN, false, 2, true>(dn_tmap, dn_smap, P.dn, smem_raw, pre_dn);
    __syncthreads();
    if (tid == 0) stream_gemm_inval(P.dn.L, smem_raw);
    __syncthreads();
    // 4. combine -> y
    layer_combine(P);
  }
  // the last CTA to finish clears the control area for the next call
  __syncthreads();
  int last = 0;
  if (tid == 0) {
    __threadfence();
    last = atomicAdd(P.ctl + 1, 1) == G - 1;
  }
  last = __syncthreads_or(last);
  if (last) {
    __threadfence();
    for (int i = tid; i < P.ctl_words; i += blockDim.x) P.ctl[i] = 0;
  }
}

}  // namespace w4

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

size_t w4_stream_workspace_bytes(int64_t rows, int N, int K, int E, int epi, bool dense, int sm_count,
                                 bool zp);

static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

// routed rows and token blocks the control area is sized for (any T of the layer's shape)
static int64_t layer_rows_max(int E, int k) {
  return std::min<int64_t>(static_cast<int64_t>(w4::kLayerMaxT) * k, 6LL * E);
}
static int64_t layer_blocks(int64_t rows, int E) {
  return std::min<int64_t>(rows, rows / 8 + std::min<int64_t>(E, rows));
}

struct LayerWs {
  int64_t nbm;              // token blocks of the control area
  size_t ctl;               // control area bytes
  size_t ids, w, offs, sorted, pos, rowblk, h, o, gu, dn, total;   // offsets of the regions
};

static LayerWs layer_ws(int T, int E, int k, int H, int I, int sm_count) {
  LayerWs L{};
  const int64_t rows = static_cast<int64_t>(T) * k;
  L.nbm = layer_blocks(layer_rows_max(E, k), E);
  const int64_t tiles_gu = (I + w4::kHalf - 1) / w4::kHalf, tiles_dn = (H + w4::kBN - 1) / w4::kBN;
  L.ctl = al256(sizeof(int32_t) * (w4::kLayerCtlHeader + 4 * L.nbm + L.nbm * (tiles_gu + tiles_dn)));
  size_t off = L.ctl;
  auto take = [&](size_t bytes) { const size_t at = off; off += al256(bytes); return at; };
  L.ids = take(sizeof(int32_t) * rows);
  L.w = take(sizeof(float) * rows);
  L.offs = take(sizeof(int32_t) * (E + 1));
  L.sorted = take(sizeof(int32_t) * rows);
  L.pos = take(sizeof(int32_t) * rows);
  L.rowblk = take(sizeof(int32_t) * rows);
  L.h = take(2 * rows * static_cast<size_t>(I));
  L.o = take(2 * rows * static_cast<size_t>(H));
  L.gu = take(w4_stream_workspace_bytes(rows, 2 * I, H, E, W4_EPI_GELU_GATE, false, sm_count, false));
  L.dn = take(w4_stream_workspace_bytes(rows, H, I, E, W4_EPI_NONE, false, sm_count, false));
  L.total = off;
  return L;
}

// W4_ERR_UNSUPPORTED outside the fused kernel's range (the four-call path covers it)
w4_status w4_layer_check(int T, int E, int k, int H, int I) {
  if (T < 0 || E < 1 || k < 1 || k > 32 || k > E || H < 32 || I < 32 || H % 32 || I % 32) return W4_ERR_INVALID_ARG;
  if (T > w4::kLayerMaxT || E > w4::kThreads || static_cast<int64_t>(T) * k > 6LL * E) return W4_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(E) * 2 * I > (1LL << 31) - 1 || static_cast<int64_t>(E) * H > (1LL << 31) - 1)
    return W4_ERR_UNSUPPORTED;
  return W4_OK;
}

size_t w4_layer_workspace_bytes(int T, int E, int k, int H, int I, int sm_count) {
  if (w4_layer_check(T, E, k, H, I) != W4_OK) return 0;
  return layer_ws(T, E, k, H, I, sm_count).total;
}

size_t w4_layer_control_bytes(int E, int k, int H, int I, int sm_count) {
  if (w4_layer_check(0, E, k, H, I) != W4_OK) return 0;
  return layer_ws(0, E, k, H, I, sm_count).ctl;
}

template <int SGU, int SDN>
static cudaError_t launch_layer(const StreamCall& gu, const StreamCall& dn, const w4::LayerArgs& P, size_t smem,
                                int sm_count, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(w4::moe_layer_kernel<SGU, SDN>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, w4::kSmemPerCta);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count);
  cfg.blockDim = dim3(w4::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the phases hand over by counters
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w4::moe_layer_kernel<SGU, SDN>, gu.tmap, gu.smap, dn.tmap, dn.smap, P);
}

w4_status w4_launch_moe_layer(const uint16_t* x, const float* logits, int T, int E, int k,
                              const uint32_t* gu_codes, const uint16_t* gu_scales, const uint32_t* dn_codes,
                              const uint16_t* dn_scales, int H, int I, uint16_t* y, void* ws, size_t ws_bytes,
                              int32_t* dev_status, cudaStream_t stream, int sm_count) {
  const w4_status chk = w4_layer_check(T, E, k, H, I);
  if (chk != W4_OK) return chk;
  if (T == 0) return W4_OK;
  const LayerWs L = layer_ws(T, E, k, H, I, sm_count);
  if (ws == nullptr || ws_bytes < L.total) return W4_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const int64_t rows = static_cast<int64_t>(T) * k;
  const int64_t tiles_gu = (I + w4::kHalf - 1) / w4::kHalf;
  int32_t* offsets = reinterpret_cast<int32_t*>(wsb + L.offs);   // written by the kernel's routing
  StreamCall gu, dn;
  // gate/up: scales by TMA or direct loads (the fused kernel keeps two scale modes per GEMM)
  w4_status st = w4_stream_setup(gu_codes, gu_scales, offsets, E, rows, 2 * I, H, W4_EPI_GELU_GATE, dev_status,
                                 sm_count, 0, -1, nullptr, 32, gu, false);
  if (st != W4_OK) return st;
  st = w4_stream_setup(dn_codes, dn_scales, offsets, E, rows, H, I, W4_EPI_NONE, dev_status, sm_count, 0, -1,
                       nullptr, 32, dn, true);
  if (st != W4_OK) return st;
  if (gu.p.MT != 8 || dn.p.MT != 8) return W4_ERR_UNSUPPORTED;
  w4_stream_bind(gu, wsb + L.gu);
  w4_stream_bind(dn, wsb + L.dn);

  w4::LayerArgs P{};
  int32_t* ctl = reinterpret_cast<int32_t*>(wsb);
  P.ctl = ctl;
  P.ctl_words = static_cast<int>(L.ctl / sizeof(int32_t));
  P.ready_gu = ctl + w4::kLayerCtlHeader;
  P.done_gu = P.ready_gu + L.nbm;
  P.ready_dn = P.done_gu + L.nbm;
  P.done_dn = P.ready_dn + L.nbm;
  int32_t* cnt_gu = P.done_dn + L.nbm;                 // split-K arrival counters
  int32_t* cnt_dn = cnt_gu + L.nbm * tiles_gu;
  P.n_blocks = gu.n_blocks;
  P.R = w4::RouteArgs{logits, T, E, k, reinterpret_cast<int32_t*>(wsb + L.ids), reinterpret_cast<float*>(wsb + L.w),
                      offsets, reinterpret_cast<int32_t*>(wsb + L.sorted),
                      reinterpret_cast<int32_t*>(wsb + L.pos), nullptr, 0, 1};
  P.row_blk = reinterpret_cast<int32_t*>(wsb + L.rowblk);
  P.x = x;
  P.y = y;
  P.H = H;
  P.I = I;
  uint16_t* h = reinterpret_cast<uint16_t*>(wsb + L.h);
  uint16_t* o = reinterpret_cast<uint16_t*>(wsb + L.o);
  // the GEMMs read the routing the kernel writes, and hand over through the control area
  gu.A.out = h;
  dn.A.out = o;
  gu.A.counters = cnt_gu;
  dn.A.counters = cnt_dn;
  gu.A.act_ready = P.ready_gu;
  gu.A.tile_done = P.done_gu;
  dn.A.act_ready = P.ready_dn;
  dn.A.tile_done = P.done_dn;
  P.gu = gu.A;
  P.dn = dn.A;
  P.dev_status = dev_status;
  P.wait_ns = w4::kWaitLimitNs;

  const size_t route_smem = (static_cast<size_t>(E) * ((T + 31) / 32) + E + static_cast<size_t>(T) * k + 32) * sizeof(int);
  const size_t smem = std::max({static_cast<size_t>(gu.A.L.total), static_cast<size_t>(dn.A.L.total), route_smem});
  if (smem > static_cast<size_t>(w4::kSmemPerCta)) return W4_ERR_UNSUPPORTED;
  cudaError_t e;
  const bool gt = gu.scale_mode == w4::kScaleTma;
  if (dn.scale_mode == w4::kScaleTma)
    e = gt ? launch_layer<w4::kScaleTma, w4::kScaleTma>(gu, dn, P, smem, sm_count, stream)
           : launch_layer<w4::kScaleLdg, w4::kScaleTma>(gu, dn, P, smem, sm_count, stream);
  else if (dn.scale_mode == w4::kScaleBlock)
    e = gt ? launch_layer<w4::kScaleTma, w4::kScaleBlock>(gu, dn, P, smem, sm_count, stream)
           : launch_layer<w4::kScaleLdg, w4::kScaleBlock>(gu, dn, P, smem, sm_count, stream);
  else
    e = gt ? launch_layer<w4::kScaleTma, w4::kScaleLdg>(gu, dn, P, smem, sm_count, stream)
           : launch_layer<w4::kScaleLdg, w4::kScaleLdg>(gu, dn, P, smem, sm_count, stream);
  return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}
