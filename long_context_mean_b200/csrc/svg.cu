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
// Those rows alone are computed (rows_attn_kernel), densely and under each
// candidate.
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

// Attention of a few query rows (the online profile's sampled rows): one
// CTA per (head, sampled row).  Its 8 warps take the key tiles in turn; in a
// warp, four groups of 8 lanes each follow every fourth key of the tile with
// their own online softmax over single keys (a lane holds d/8 consecutive
// dimensions, read as 16-byte vectors), and the 32 partial states are merged
// at the end.  Dense: every key.  Candidate: the keys of the kept tiles of
// the row's query block in head h's order (perms[h][place] = token at that
// place; block_mask[h][qb][kb]).
constexpr int kRowsWarps = 8;
constexpr int kRowsGroups = 4;                 // lane groups per warp
constexpr int kRowsStates = kRowsWarps * kRowsGroups;
constexpr int kRowsMaxTiles = 4096;

template <typename T, int D>
__global__ void __launch_bounds__(32 * kRowsWarps) rows_attn_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int64_t Hq, int64_t Hkv, int64_t N,
    const int32_t* __restrict__ rows, int64_t nrows, const int32_t* __restrict__ perms,
    const uint8_t* __restrict__ block_mask, int bq, int bk, int64_t nqb, int64_t nkb, float scale_log2,
    float* __restrict__ out, float* __restrict__ lse, int32_t* status) {
  constexpr int EPV = 16 / (int)sizeof(T);     // elements per 16-byte vector
  constexpr int DL = D / 8;                    // dimensions per lane
  constexpr int VL = DL / EPV;                 // vectors per lane
  static_assert(VL >= 1 && DL % EPV == 0, "d / 8 must fill whole 16-byte vectors");
  const int64_t bh = blockIdx.x / nrows, r = blockIdx.x % nrows;
  const int64_t b = bh / Hq, h = bh % Hq, kvh = b * Hkv + h / (Hq / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, gl = lane & 7;
  __shared__ int32_t s_place, s_ntiles;
  __shared__ int32_t s_tiles[kRowsMaxTiles];
  __shared__ float s_m[kRowsStates], s_l[kRowsStates];
  __shared__ float s_o[kRowsStates][D];
  const int64_t i = __ldg(rows + r);
  if (i < 0 || i >= N) {                                   // uniform over the CTA
    if (threadIdx.x == 0) raise_status(status, SA_ERR_INVALID_ARG);
    return;
  }
  const int32_t* perm = perms ? perms + bh * N : nullptr;
  if (threadIdx.x == 0) s_place = perm ? -1 : (int32_t)i;
  __syncthreads();
  if (perm) {
    for (int64_t n = threadIdx.x; n < N; n += 32 * kRowsWarps)
      if (__ldg(perm + n) == i) s_place = (int32_t)n;
    __syncthreads();
    if (s_place < 0) {                                     // perms[h] is not a permutation
      if (threadIdx.x == 0) raise_status(status, SA_ERR_INVALID_ARG);
      return;
    }
  }
  if (block_mask) {
    const uint8_t* mrow = block_mask + (bh * nqb + s_place / bq) * nkb;
    if (warp == 0) {
      int cnt = 0;
      for (int64_t kb0 = 0; kb0 < nkb; kb0 += 32) {
        const int64_t kb = kb0 + lane;
        const bool kept = kb < nkb && __ldg(mrow + kb) != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, kept);
        if (kept) s_tiles[cnt + __popc(bal & ((1u << lane) - 1u))] = (int32_t)kb;
        cnt += __popc(bal);
      }
      if (lane == 0) s_ntiles = cnt;
    }
  } else {
    for (int64_t kb = threadIdx.x; kb < nkb; kb += 32 * kRowsWarps) s_tiles[kb] = (int32_t)kb;
    if (threadIdx.x == 0) s_ntiles = (int32_t)nkb;
  }
  float qv[DL];
  {
    const uint4* qp = reinterpret_cast<const uint4*>(q + (bh * N + i) * D + gl * DL);
#pragma unroll
    for (int c = 0; c < VL; ++c) unpack16(__ldg(qp + c), T(), qv + c * EPV);
#pragma unroll
    for (int e = 0; e < DL; ++e) qv[e] *= scale_log2;
  }
  __syncthreads();
  const int ntiles = s_ntiles;
  const T* kh = k + kvh * N * D + gl * DL;
  const T* vh = v + kvh * N * D + gl * DL;
  float m = -INFINITY, l = 0.f, o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = 0.f;
  for (int t = warp; t < ntiles; t += kRowsWarps) {
    const int64_t j0 = (int64_t)s_tiles[t] * bk, j1 = min64(N, j0 + bk);
    for (int64_t jj = j0; jj < j1; jj += kRowsGroups) {    // uniform over the warp
      const int64_t j = jj + grp;
      int64_t key = j < j1 ? (perm ? (int64_t)__ldg(perm + j) : j) : j0;
      // An entry of perms outside [0, N) (not a permutation) is reported and
      // left out, as the pooling pass does.
      const bool in_range = (uint64_t)key < (uint64_t)N;
      if (j < j1 && !in_range) raise_status(status, SA_ERR_INVALID_ARG);
      const bool valid = j < j1 && in_range;
      if (!in_range) key = j0;
      const uint4* kp = reinterpret_cast<const uint4*>(kh + key * D);
      const uint4* vp = reinterpret_cast<const uint4*>(vh + key * D);
      float kf[DL], vf[DL];
#pragma unroll
      for (int c = 0; c < VL; ++c) unpack16(__ldg(kp + c), T(), kf + c * EPV);
#pragma unroll
      for (int c = 0; c < VL; ++c) unpack16(__ldg(vp + c), T(), vf + c * EPV);
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < DL; ++e) s = fmaf(qv[e], kf[e], s);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      if (valid) {
        const float mn = fmaxf(m, s);
        const float corr = exp2f(m - mn), p = exp2f(s - mn);
        l = fmaf(l, corr, p);
#pragma unroll
        for (int e = 0; e < DL; ++e) o[e] = fmaf(p, vf[e], o[e] * corr);
        m = mn;
      }
    }
  }
  const int sid = warp * kRowsGroups + grp;
  if (gl == 0) {
    s_m[sid] = m;
    s_l[sid] = l;
  }
#pragma unroll
  for (int e = 0; e < DL; ++e) s_o[sid][gl * DL + e] = o[e];
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int w = 0; w < kRowsStates; ++w) M = fmaxf(M, s_m[w]);
    float L = 0.f, O[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) O[e] = 0.f;
    for (int w = 0; w < kRowsStates; ++w) {
      const float f = s_m[w] > -INFINITY ? exp2f(s_m[w] - M) : 0.f;
      L = fmaf(s_l[w], f, L);
#pragma unroll
      for (int e = 0; e < D / 32; ++e) O[e] = fmaf(s_o[w][lane + 32 * e], f, O[e]);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) out[(bh * nrows + r) * D + lane + 32 * e] = O[e] * inv;
    if (lane == 0) {
      if (!(L > 0.f)) raise_status(status, SA_ERR_EMPTY_ROW);
      if (lse) lse[bh * nrows + r] = (M + log2f(L)) * 0.6931471805599453f;
    }
  }
}

}  // namespace

bool rows_attn_supported(int64_t d, int64_t dv, int64_t N, int bk) {
  return d == dv && (d == 64 || d == 128) && ceil_div(N, bk) <= kRowsMaxTiles;
}

sa_status launch_rows_attn(const void* q, const void* k, const void* v, const sa_shape& s, const int32_t* rows,
                           int64_t nrows, const int32_t* perms, const uint8_t* block_mask, int bq, int bk,
                           float scale, float* out, float* lse, int32_t* status, cudaStream_t st) {
  const int64_t BH = s.B * s.Hq;
  if (BH == 0 || nrows == 0) return SA_OK;
  if (BH * nrows > 2147483647) return set_error(SA_ERR_UNSUPPORTED, "too many rows");
  const int64_t nqb = ceil_div(s.N, bq), nkb = ceil_div(s.N, bk);
  const float sl2 = scale * 1.4426950408889634f;
  const unsigned grid = (unsigned)(BH * nrows);
#define SA_ROWS_LAUNCH(T, D)                                                                                \
  rows_attn_kernel<T, D><<<grid, 32 * kRowsWarps, 0, st>>>(                                                 \
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), s.Hq, s.Hkv, s.N, rows,   \
      nrows, perms, block_mask, bq, bk, nqb, nkb, sl2, out, lse, status)
#define SA_ROWS_D(T)                  \
  switch (s.d) {                      \
    case 64: SA_ROWS_LAUNCH(T, 64); break; \
    default: SA_ROWS_LAUNCH(T, 128); break; \
  }
  if (s.dtype == SA_BF16) {
    SA_ROWS_D(uint16_t)
  } else {
    SA_ROWS_D(float)
  }
#undef SA_ROWS_D
#undef SA_ROWS_LAUNCH
  return check_launch("rows_attn_kernel");
}

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
