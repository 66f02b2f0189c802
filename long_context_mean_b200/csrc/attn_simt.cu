// Portable CUDA-core block-sparse attention: the reference kernel for shapes
// the tensor-core kernel does not serve (fp32, d != 128, small blocks) and a
// second, independent GPU path for testing.
//
// [P3] SpargeAttention notes 2.1: for each query block, visit the kept key
// blocks; S = Q K^T * scale; m_new = max(m, rowmax S); P = exp(S - m_new);
// l = exp(m - m_new) l + rowsum P; O = exp(m - m_new) O + P V; finally O / l.
// 2.3: skip P V for the tile when the largest (rowmax S - m_new) over the
// block's rows is < lambda (the normaliser still counts the tile; every
// row's maximum is then unchanged, so O needs no rescale).
#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int bq = a.bq, bk = a.bk;
  const int dv = (int)a.dv, d = (int)a.d;
  float* O = sm;                    // [bq][dv]
  float* S = O + bq * dv;           // [bq][bk]
  float* m = S + bq * bk;           // [bq]
  float* l = m + bq;                // [bq]
  float* corr = l + bq;             // [bq]
  __shared__ float red[kThreads / 32];
  __shared__ int s_skip;

  const int64_t u = a.order ? a.order[blockIdx.x] : blockIdx.x;
  const int64_t bh = u / a.nqb, qb = u % a.nqb;
  const int64_t b = bh / a.Hq, h = bh % a.Hq;
  const int64_t kvh = b * a.Hkv + h / (a.Hq / a.Hkv);
  const T* q = static_cast<const T*>(a.q) + bh * a.N * d;
  const T* k = static_cast<const T*>(a.k) + kvh * a.N * d;
  const T* v = static_cast<const T*>(a.v) + kvh * a.N * dv;
  const int64_t i0 = qb * bq;
  const int nr = (int)min64(bq, a.N - i0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  for (int i = threadIdx.x; i < nr * dv; i += kThreads) O[i] = 0.f;
  for (int r = threadIdx.x; r < nr; r += kThreads) {
    m[r] = -INFINITY;
    l[r] = 0.f;
  }

  int64_t lo = 0, hi;
  if (a.row_ptr) {
    lo = a.row_ptr[u];
    hi = a.row_ptr[u + 1];
    if (hi > a.col_capacity || lo > hi) {
      // The list reaches past col_idx: the builder raised SA_ERR_CAPACITY;
      // the row is not computed.
      if (threadIdx.x == 0) raise_status(a.status, SA_ERR_CAPACITY);
      return;
    }
  } else {
    const int64_t last_row = i0 + nr - 1;
    hi = a.causal ? (last_row / bk + 1) : a.nkb;
  }
  __syncthreads();

  for (int64_t t = lo; t < hi; ++t) {
    const int64_t kb = a.row_ptr ? a.col_idx[t] : t;
    if (kb < 0 || kb >= a.nkb) {   // not a list a mask builder wrote
      if (threadIdx.x == 0) raise_status(a.status, SA_ERR_INVALID_ARG);
      continue;
    }
    const int64_t j0 = kb * bk;
    const int nc = (int)min64(bk, a.N - j0);
    // Scores.
    for (int idx = threadIdx.x; idx < nr * nc; idx += kThreads) {
      const int r = idx / nc, j = idx % nc;
      const T* qr = q + (i0 + r) * d;
      const T* kr = k + (j0 + j) * d;
      float acc = 0.f;
      for (int e = 0; e < d; ++e) acc = fmaf(Elem<T>::load(qr + e), Elem<T>::load(kr + e), acc);
      float s = acc * a.scale;
      if (a.causal && j0 + j > i0 + r) s = -INFINITY;
      S[r * bk + j] = s;
    }
    __syncthreads();
    // Row statistics, one warp per row.
    float gmax = -INFINITY;
    for (int r = warp; r < nr; r += kThreads / 32) {
      float mloc = -INFINITY;
      for (int j = lane; j < nc; j += 32) mloc = fmaxf(mloc, S[r * bk + j]);
      for (int off = 16; off > 0; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
      const float mold = m[r];
      const float mnew = fmaxf(mold, mloc);
      float rs = 0.f;
      for (int j = lane; j < nc; j += 32) {
        const float s = S[r * bk + j];
        const float p = (s == -INFINITY) ? 0.f : expf(s - mnew);
        S[r * bk + j] = p;
        rs += p;
      }
      for (int off = 16; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
      if (lane == 0) {
        const float c = (mnew == -INFINITY) ? 1.f : (mold == -INFINITY ? 0.f : expf(mold - mnew));
        corr[r] = c;
        l[r] = c * l[r] + rs;
        m[r] = mnew;
      }
      if (mloc > -INFINITY) gmax = fmaxf(gmax, mloc - mnew);
    }
    for (int off = 16; off > 0; off >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, off));
    if (lane == 0) red[warp] = gmax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float g = -INFINITY;
      for (int w = 0; w < kThreads / 32; ++w) g = fmaxf(g, red[w]);
      const int skip = g < a.lambda ? 1 : 0;
      s_skip = skip;
      if (a.skip_log) a.skip_log[t] = (uint8_t)skip;
    }
    __syncthreads();
    if (!s_skip) {
      for (int idx = threadIdx.x; idx < nr * dv; idx += kThreads) {
        const int r = idx / dv, c = idx % dv;
        float acc = 0.f;
        for (int j = 0; j < nc; ++j) acc = fmaf(S[r * bk + j], Elem<T>::load(v + (j0 + j) * dv + c), acc);
        O[idx] = corr[r] * O[idx] + acc;
      }
    }
    __syncthreads();
  }

  T* out = static_cast<T*>(a.out) + bh * a.N * dv;
  for (int idx = threadIdx.x; idx < nr * dv; idx += kThreads) {
    const int r = idx / dv, c = idx % dv;
    const float lr = l[r];
    const int64_t orow = a.out_perm ? a.out_perm[bh * a.perm_stride + i0 + r] : i0 + r;
    Elem<T>::store(out + orow * dv + c, lr > 0.f ? O[idx] / lr : 0.f);
  }
  for (int r = threadIdx.x; r < nr; r += kThreads) {
    if (!(l[r] > 0.f)) raise_status(a.status, SA_ERR_EMPTY_ROW);
    const int64_t orow = a.out_perm ? a.out_perm[bh * a.perm_stride + i0 + r] : i0 + r;
    if (a.lse) a.lse[bh * a.N + orow] = m[r] + logf(l[r]);
  }
}

}  // namespace

sa_status launch_attn_simt(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = ((size_t)a.bq * a.dv + (size_t)a.bq * a.bk + 3 * (size_t)a.bq) * 4;
  if (smem > 227 * 1024) return set_error(SA_ERR_UNSUPPORTED, "bq*dv + bq*bk too large for the CUDA-core kernel");
  const int64_t R = a.B * a.Hq * a.nqb;
  if (R == 0) return SA_OK;
  if (a.dtype == SA_BF16) {
    if (cudaFuncSetAttribute(attn_simt_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(attn_simt_kernel) failed");
    attn_simt_kernel<uint16_t><<<(unsigned)R, kThreads, smem, st>>>(a);
  } else {
    if (cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(attn_simt_kernel) failed");
    attn_simt_kernel<float><<<(unsigned)R, kThreads, smem, st>>>(a);
  }
  return check_launch("attn_simt_kernel");
}

}  // namespace sa
