// Per-head placement of fixed spatial and temporal masks, and the
// sampled-row output error that chooses between them: the Sparse VideoGen
// comparison of [P1] ("AIGC 基本功｜视频稀疏注意力的误差与布局", sections
// 3.3, 3.4, 4 and 5).
//
// A spatial head keeps the (query, key) pairs of one frame, a temporal head
// the pairs of one spatial position across frames; text tokens (after the
// nv = T*P video tokens, P = H*W) see and are seen by every token.  A
// spatial head runs in the frame-major order (token t*P + p, the identity);
// a temporal head in the token-major order (position p = n / T, frame
// t = n % T at place n < nv; text in place), where a position's pairs are
// contiguous.  In its own order a video token's group (frame or position)
// is its index divided by the group size (P or T), so a (query block, key
// block) tile holds an allowed pair iff it reaches a text token or the two
// blocks' group ranges intersect: the block mask is the block-level cover
// of the element mask (the tile ledger of section 4).
//
// The selection compares each candidate's output with dense attention on a
// few sampled query rows: the mean squared error over those rows' outputs.
#include "sa_internal.cuh"

namespace sa {
namespace {

// perms[h][n] = source token of place n for head h; mask[h][qb][kb] = the
// tile cover.  kinds[h]: 0 spatial, 1 temporal; anything else raises
// SA_ERR_INVALID_ARG and leaves the head's tiles empty (identity order).
__global__ void __launch_bounds__(256) head_placement_kernel(int64_t T, int64_t P, int64_t n,
                                                             const int32_t* __restrict__ kinds, int64_t heads,
                                                             int bq, int bk, int64_t nqb, int64_t nkb,
                                                             int32_t* __restrict__ perms,
                                                             uint8_t* __restrict__ mask, int32_t* status) {
  const int64_t nv = T * P;
  const int64_t step = (int64_t)gridDim.x * blockDim.x;
  const int64_t first = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (perms) {
    for (int64_t e = first; e < heads * n; e += step) {
      const int64_t h = e / n, i = e % n;
      const int32_t kind = __ldg(kinds + h);
      perms[e] = (int32_t)(kind == SA_HEAD_TEMPORAL && i < nv ? (i % T) * P + i / T : i);
    }
  }
  if (mask) {
    const int64_t tiles = nqb * nkb;
    for (int64_t e = first; e < heads * tiles; e += step) {
      const int64_t h = e / tiles, t = e % tiles;
      const int32_t kind = __ldg(kinds + h);
      if (kind != SA_HEAD_SPATIAL && kind != SA_HEAD_TEMPORAL) {
        if (t == 0) raise_status(status, SA_ERR_INVALID_ARG);
        mask[e] = 0;
        continue;
      }
      const int64_t group = kind == SA_HEAD_SPATIAL ? P : T;
      const int64_t qb = t / nkb, kb = t % nkb;
      const int64_t i0 = qb * bq, i1 = min64(n, (qb + 1) * bq) - 1;   // places of the query block
      const int64_t j0 = kb * bk, j1 = min64(n, (kb + 1) * bk) - 1;   // places of the key block
      const bool keep = i1 >= nv || j1 >= nv ||                        // a text token is involved
                        (i0 / group <= j1 / group && j0 / group <= i1 / group);
      mask[e] = keep ? 1 : 0;
    }
  }
}

// out[h] = mean over the sampled rows r and the dv outputs of (ref - x)^2.
template <typename T>
__global__ void __launch_bounds__(256) rows_mse_kernel(const T* __restrict__ ref, const T* __restrict__ x,
                                                       const int32_t* __restrict__ rows, int64_t nrows, int64_t N,
                                                       int64_t dv, double* __restrict__ out, int32_t* status) {
  const int64_t h = blockIdx.x;
  double acc = 0.0;
  for (int64_t e = threadIdx.x; e < nrows * dv; e += blockDim.x) {
    const int64_t r = __ldg(rows + e / dv);
    if (r < 0 || r >= N) {
      raise_status(status, SA_ERR_INVALID_ARG);
      continue;
    }
    const int64_t off = (h * N + r) * dv + e % dv;
    const double diff = (double)Elem<T>::load(ref + off) - (double)Elem<T>::load(x + off);
    acc += diff * diff;
  }
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[h] = nrows > 0 ? red[0] / (double)(nrows * dv) : 0.0;
}

}  // namespace

sa_status launch_head_placement(int64_t T, int64_t P, int64_t n, const int32_t* kinds, int64_t heads, int bq,
                                int bk, int32_t* perms, uint8_t* mask, int32_t* status, cudaStream_t st) {
  const int64_t nqb = ceil_div(n, bq), nkb = ceil_div(n, bk);
  const int64_t per_mask = mask ? nqb * nkb : 0, per_perm = perms ? n : 0;
  const int64_t work = heads * (per_mask > per_perm ? per_mask : per_perm);
  if (work == 0) return SA_OK;
  const int grid = (int)min64(ceil_div(work, 256), 148 * 8);
  head_placement_kernel<<<grid, 256, 0, st>>>(T, P, n, kinds, heads, bq, bk, nqb, nkb, perms, mask, status);
  return check_launch("head_placement_kernel");
}

sa_status launch_rows_mse(const void* ref, const void* x, const int32_t* rows, int64_t nrows, int64_t BH, int64_t N,
                          int64_t dv, int32_t dtype, double* out, int32_t* status, cudaStream_t st) {
  if (BH == 0) return SA_OK;
  if (dtype == SA_BF16)
    rows_mse_kernel<uint16_t><<<(unsigned)BH, 256, 0, st>>>(static_cast<const uint16_t*>(ref),
                                                            static_cast<const uint16_t*>(x), rows, nrows, N, dv,
                                                            out, status);
  else
    rows_mse_kernel<float><<<(unsigned)BH, 256, 0, st>>>(static_cast<const float*>(ref),
                                                         static_cast<const float*>(x), rows, nrows, N, dv, out,
                                                         status);
  return check_launch("rows_mse_kernel");
}

}  // namespace sa
