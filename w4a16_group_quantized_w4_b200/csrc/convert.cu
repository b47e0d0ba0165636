// Conversion pass in front of the tensor-core GEMMs: activations to fp16 with a power-of-two
// exponent per row, gathered into routed-pair order.
//
// Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
// "What changed in vLLM's TPU backend" (activations stay 16-bit).  fp16 with a per-row exponent
// holds every bf16 activation within 2^31 of its row's largest exactly, so the tensor-core
// products stay the exact a * s * q.
#include "tcgen05.cuh"

namespace w4 {
namespace cv {

// One warp per output row p: the activation row it reads (row p of `a`, or row
// a_row_of_pair[p] / k_div when rows are gathered) is scanned for its largest finite |a|, which
// picks f so that it lands in [2^14, 2^15); row p of a16 becomes fp16(a * 2^f) and rowmul[p] = 2^-f.
// Within every 8 consecutive k the values are stored in the order 0, 4, 1, 5, 2, 6, 3, 7: the
// order in which the GEMM extracts the nibbles of a layout-L1 code word.
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
    // lane l holds chunks l, l + 32, ... of up to kCB * 32 chunks at a time, all loads in
    // flight together; a row of at most kCB * 256 elements (K <= 3072) is read once
    constexpr int kCB = 12;
    uint4 v[kCB];
    uint32_t m = 0;
    for (int i0 = 0; i0 < nv; i0 += 32 * kCB) {
#pragma unroll
      for (int t = 0; t < kCB; ++t) {
        const int i = i0 + 32 * t + lane;
        v[t] = i < nv ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int t = 0; t < kCB; ++t) {
        const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
          if (lo < 0x7F80u) m = max(m, lo);
          if (hi < 0x7F80u) m = max(m, hi);
        }
      }
    }
    m = __reduce_max_sync(0xffffffffu, m);
    const int f = shift_for(m, 14);
    const float mul = pow2f(f);
    uint4* dst = reinterpret_cast<uint4*>(a16 + row * K);
    for (int i0 = 0; i0 < nv; i0 += 32 * kCB) {
      if (nv > 32 * kCB) {                       // long rows: the batch again (from L1 / L2)
#pragma unroll
        for (int t = 0; t < kCB; ++t) {
          const int i = i0 + 32 * t + lane;
          v[t] = i < nv ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int t = 0; t < kCB; ++t) {
        const int i = i0 + 32 * t + lane;
        if (i >= nv) break;
        const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
        uint32_t o[4];
        f16_pairs_l1(w, mul, mul, o);            // k order of the dequantised weight pairs
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    if (lane == 0) rowmul[row] = pow2f(-f);
  }
}

// Per weight row (one thread each): the exponent e that brings the row's largest finite scale
// to [2^10, 2^11), as in the dequantisation of tm_gemm.cu.  Rows of kg bf16 scales, kg even (4-byte
// aligned words).
__global__ void __launch_bounds__(256)
row_exp_kernel(const uint16_t* __restrict__ scales, int64_t wrows, int kg, int8_t* __restrict__ e_out) {
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < wrows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t* row = reinterpret_cast<const uint32_t*>(scales + r * kg);
    uint32_t m = 0;
    for (int j = 0; j < (kg >> 1); ++j) {
      const uint32_t v = __ldg(row + j);
      const uint32_t lo = v & 0x7FFFu, hi = (v >> 16) & 0x7FFFu;
      if (lo < 0x7F80u) m = max(m, lo);
      if (hi < 0x7F80u) m = max(m, hi);
    }
    e_out[r] = static_cast<int8_t>(shift_for(m, 10));
  }
}

// Short rows (at most 128 16-byte chunks, K <= 1024): a warp converts 12 / CPL rows at a time,
// lane l holding chunks l + 32 t (t < CPL) of each, so that twelve loads per lane are in flight
// as for long rows (one row per warp would leave a K = 704 row at three).  Same arithmetic as
// a_to_f16_kernel.
template <int CPL>
__global__ void __launch_bounds__(256)
a_to_f16_short_kernel(const uint16_t* __restrict__ a, const int32_t* __restrict__ a_row_of_pair,
                      int k_div, int64_t a_rows, int64_t rows, int K, uint16_t* __restrict__ a16,
                      float* __restrict__ rowmul, int32_t* dev_status) {
  constexpr int kRW = 12 / CPL;
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int nv = K >> 3;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * wpb;
  for (int64_t r0 = (blockIdx.x * wpb + (threadIdx.x >> 5)) * kRW; r0 < rows; r0 += nw * kRW) {
    uint4 v[kRW][CPL];
#pragma unroll
    for (int j = 0; j < kRW; ++j) {
      const int64_t row = r0 + j;
      int64_t srow = row;
      if (row < rows && a_row_of_pair) {
        srow = __ldg(a_row_of_pair + row) / k_div;
        if (srow < 0 || srow >= a_rows) {
          if (lane == 0) set_status(dev_status, W4_ERR_INVALID_ARG);
          srow = 0;
        }
      }
      const uint4* src = reinterpret_cast<const uint4*>(a + srow * K);
#pragma unroll
      for (int t = 0; t < CPL; ++t) {
        const int i = 32 * t + lane;
        v[j][t] = (row < rows && i < nv) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < kRW; ++j) {
      const int64_t row = r0 + j;
      uint32_t m = 0;
#pragma unroll
      for (int t = 0; t < CPL; ++t) {
        const uint32_t w[4] = {v[j][t].x, v[j][t].y, v[j][t].z, v[j][t].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = w[q] & 0x7FFFu, hi = (w[q] >> 16) & 0x7FFFu;
          if (lo < 0x7F80u) m = max(m, lo);
          if (hi < 0x7F80u) m = max(m, hi);
        }
      }
      m = __reduce_max_sync(0xffffffffu, m);
      if (row >= rows) continue;                 // the same for every lane of the warp
      const int f = shift_for(m, 14);
      const float mul = pow2f(f);
      uint4* dst = reinterpret_cast<uint4*>(a16 + row * K);
#pragma unroll
      for (int t = 0; t < CPL; ++t) {
        const int i = 32 * t + lane;
        if (i < nv) {
          const uint32_t w[4] = {v[j][t].x, v[j][t].y, v[j][t].z, v[j][t].w};
          uint32_t o[4];
          f16_pairs_l1(w, mul, mul, o);
          dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      if (lane == 0) rowmul[row] = pow2f(-f);
    }
  }
}

}  // namespace cv
}  // namespace w4

// fp16 activation rows in pair order [rows, K] (256-byte aligned), then the row multipliers
// [rows] (256-byte aligned), then the weight-row exponents [wrows] (int8)
static size_t a16_bytes(int64_t rows, int K) { return (static_cast<size_t>(rows) * K * 2 + 255) / 256 * 256; }
static size_t rowmul_bytes(int64_t rows) { return (static_cast<size_t>(rows) * 4 + 255) / 256 * 256; }

size_t w4_tc_workspace_bytes(int64_t rows, int K, int64_t wrows) {
  if (rows <= 0) return 0;
  return a16_bytes(rows, K) + rowmul_bytes(rows) + static_cast<size_t>(wrows);
}

uint16_t* w4_ws_a16(void* ws) { return static_cast<uint16_t*>(ws); }

float* w4_ws_rowmul(void* ws, int64_t rows, int K) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + a16_bytes(rows, K));
}

int8_t* w4_ws_rowexp(void* ws, int64_t rows, int K) {
  return reinterpret_cast<int8_t*>(static_cast<uint8_t*>(ws) + a16_bytes(rows, K) + rowmul_bytes(rows));
}

void w4_launch_a_to_f16(const uint16_t* a, const int32_t* a_row_of_pair, int k_div, int64_t a_rows,
                        int64_t rows, int K, const uint16_t* scales, int64_t wrows, void* ws,
                        int32_t* dev_status, cudaStream_t stream, int sm_count) {
  if (rows <= 0) return;
  const int nv = K >> 3;
  if (nv <= 128) {
    // short rows: 12 / cpl rows per warp at a time
    const int cpl = (nv + 31) / 32;
    const int64_t warps = (rows + 12 / cpl - 1) / (12 / cpl);
    const int64_t blocks = (warps + 7) / 8;
    const int grid = static_cast<int>(blocks < 16LL * sm_count ? blocks : 16LL * sm_count);
    uint16_t* a16 = w4_ws_a16(ws);
    float* rm = w4_ws_rowmul(ws, rows, K);
    switch (cpl) {
      case 1: w4::cv::a_to_f16_short_kernel<1><<<grid, 256, 0, stream>>>(a, a_row_of_pair, k_div, a_rows, rows, K, a16, rm, dev_status); break;
      case 2: w4::cv::a_to_f16_short_kernel<2><<<grid, 256, 0, stream>>>(a, a_row_of_pair, k_div, a_rows, rows, K, a16, rm, dev_status); break;
      case 3: w4::cv::a_to_f16_short_kernel<3><<<grid, 256, 0, stream>>>(a, a_row_of_pair, k_div, a_rows, rows, K, a16, rm, dev_status); break;
      default: w4::cv::a_to_f16_short_kernel<4><<<grid, 256, 0, stream>>>(a, a_row_of_pair, k_div, a_rows, rows, K, a16, rm, dev_status); break;
    }
  } else {
    const int64_t blocks = (rows + 7) / 8;
    const int grid = static_cast<int>(blocks < 16LL * sm_count ? blocks : 16LL * sm_count);
    w4::cv::a_to_f16_kernel<<<grid, 256, 0, stream>>>(a, a_row_of_pair, k_div, a_rows, rows, K,
                                                      w4_ws_a16(ws), w4_ws_rowmul(ws, rows, K),
                                                      dev_status);
  }
  if (wrows > 0) {
    const int64_t eb = (wrows + 255) / 256;
    const int egrid = static_cast<int>(eb < 8LL * sm_count ? eb : 8LL * sm_count);
    w4::cv::row_exp_kernel<<<egrid, 256, 0, stream>>>(scales, wrows, K / 32, w4_ws_rowexp(ws, rows, K));
  }
}
