// Per-block 8-bit quantisation of Q and K for the quantised QK path of the
// SpargeAttention notes ([P3] section 2.4: the QK product runs on
// SageAttention's per-block quantisation with dequantisation scales).
//
// A block is `rows` consecutive tokens of one head over all d channels
// (the query block for Q, the key block for K).  INT8: scale absmax / 127,
// every value becomes rint(x * (127 / absmax)) computed in float32 (round
// half to even), in [-127, 127].  FP8 E4M3: scale absmax / 448, every value
// becomes the E4M3 value nearest to x * (448 / absmax) (float32 product,
// hardware conversion: ties to even, saturated to +-448).  An all-zero block
// has scale 0 and codes 0.  Both divisions are correctly rounded
// (__fdiv_rn), so the codes do not depend on compiler flags.
//
// The attention kernel multiplies the tile of q8 . k8 (exact int32 for
// INT8, fp32-accumulated for E4M3) by one float per kept tile:
// scale * log2(e) * scale_q(query block) * scale_k(key block), written in
// CSR order by tile_scales_kernel.
#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantMaxVec = 8;   // 16-byte vectors per thread: rows * d <= 256 * 8 * 8

__device__ __forceinline__ uint32_t bf16_abs_max4(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = max(m, w[i] & 0x7FFFu);
    m = max(m, (w[i] >> 16) & 0x7FFFu);
  }
  return m;
}

// One CTA per (head, block).  x: bf16 [heads][N][d]; x8: 8-bit codes
// [heads][N][d]; scales: float [heads][nblk].
template <int FMT>
__global__ void __launch_bounds__(kQuantThreads) quant_blocks_kernel(const uint4* __restrict__ x, int64_t N, int d,
                                                                     int rows, int64_t nblk, uint2* __restrict__ x8,
                                                                     float* __restrict__ scales) {
  const int64_t h = blockIdx.x / nblk, b = blockIdx.x % nblk;
  const int64_t r0 = b * rows;
  const int64_t nr = min64(rows, N - r0);
  const int vpr = d / 8;
  const int64_t total = nr * vpr;
  const int64_t base = (h * N + r0) * vpr;           // in 16-byte vectors of 8 values
  uint4 v[kQuantMaxVec];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kQuantMaxVec; ++i) {
    const int64_t e = threadIdx.x + (int64_t)i * kQuantThreads;
    if (e < total) {
      v[i] = __ldg(x + base + e);
      m = max(m, bf16_abs_max4(v[i]));
    }
  }
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t wmax[kQuantThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  m = 0;
#pragma unroll
  for (int w = 0; w < kQuantThreads / 32; ++w) m = max(m, wmax[w]);
  const float amax = __uint_as_float(m << 16);
  const float qmax = FMT == SA_Q_E4M3 ? 448.0f : 127.0f;
  const float inv = amax > 0.f ? __fdiv_rn(qmax, amax) : 0.f;
  if (threadIdx.x == 0) scales[blockIdx.x] = amax > 0.f ? __fdiv_rn(amax, qmax) : 0.f;
#pragma unroll
  for (int i = 0; i < kQuantMaxVec; ++i) {
    const int64_t e = threadIdx.x + (int64_t)i * kQuantThreads;
    if (e < total) {
      x8[base + e] = quant8<FMT>(v[i], inv);
    }
  }
}

// ts[e] = scale_log2 * q_scales[row] * k_scales[kv head][col_idx[e]] for
// every list entry e of row (bh, qb); one warp per row.  A row whose list
// reaches past the capacity of col_idx (and of ts) is left out: the mask's
// builder has raised SA_ERR_CAPACITY for it.
__global__ void __launch_bounds__(256) tile_scales_kernel(const int32_t* __restrict__ row_ptr,
                                                          const int32_t* __restrict__ col_idx, int64_t R,
                                                          int64_t capacity, int64_t nqb, int64_t nkb,
                                                          int64_t Hq, int64_t Hkv,
                                                          const float* __restrict__ qs, const float* __restrict__ ks,
                                                          float scale_log2, float* __restrict__ ts) {
  const int64_t r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const int64_t bh = r / nqb, b = bh / Hq, h = bh % Hq;
  const int64_t kvh = b * Hkv + h / (Hq / Hkv);
  const float a = scale_log2 * __ldg(qs + r);
  const float* kr = ks + kvh * nkb;
  const int32_t e1 = __ldg(row_ptr + r + 1);
  if (e1 > capacity) return;
  for (int32_t e = __ldg(row_ptr + r) + lane; e < e1; e += 32) {
    const int32_t kb = __ldg(col_idx + e);
    ts[e] = (kb >= 0 && kb < nkb) ? a * __ldg(kr + kb) : 0.f;
  }
}

}  // namespace

sa_status launch_quant_blocks(const void* x, int64_t heads, int64_t N, int64_t d, int rows, int32_t fmt, void* x8,
                              float* scales, cudaStream_t st) {
  const int64_t nblk = ceil_div(N, rows);
  const int64_t ctas = heads * nblk;
  if (ctas == 0) return SA_OK;
  if (ctas > 2147483647) return set_error(SA_ERR_UNSUPPORTED, "too many blocks");
  if (fmt == SA_Q_E4M3)
    quant_blocks_kernel<SA_Q_E4M3><<<(unsigned)ctas, kQuantThreads, 0, st>>>(
        static_cast<const uint4*>(x), N, (int)d, rows, nblk, static_cast<uint2*>(x8), scales);
  else
    quant_blocks_kernel<SA_Q_INT8><<<(unsigned)ctas, kQuantThreads, 0, st>>>(
        static_cast<const uint4*>(x), N, (int)d, rows, nblk, static_cast<uint2*>(x8), scales);
  return check_launch("quant_blocks_kernel");
}

bool quant_blocks_fits(int64_t d, int rows) { return d % 8 == 0 && (int64_t)rows * d <= 8LL * kQuantThreads * kQuantMaxVec; }

sa_status launch_tile_scales(const sa_mask& m, int64_t B, int64_t Hq, int64_t Hkv, const float* qs, const float* ks,
                             float scale_log2, float* ts, cudaStream_t st) {
  const int64_t R = B * Hq * m.nqb;
  if (R == 0) return SA_OK;
  tile_scales_kernel<<<(unsigned)ceil_div(R, 8), 256, 0, st>>>(m.row_ptr, m.col_idx, R, m.col_capacity, m.nqb,
                                                               m.nkb, Hq, Hkv, qs, ks, scale_log2, ts);
  return check_launch("tile_scales_kernel");
}

}  // namespace sa
