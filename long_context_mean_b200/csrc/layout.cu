// Token layouts and the reorder / inverse reorder of row-major token tensors.
//
// Layouts ([P2] MindIE-SD "稀疏": [t,h,w] window reorder with the first frame
// kept as a sink; [P3] SpargeAttention notes 2.5: Hilbert-curve permutation
// of the visual tokens, inverse permutation on the output; [P1] 3.4: the
// same permutation applied to Q, K, V and undone on O leaves the attention
// result unchanged).
//
// perm[n] is the source index of output position n, inv the inverse.
#include "sa_internal.cuh"

namespace sa {
namespace {

// ---------------------------------------------------------------------------
// Window layout: each thread places one source token in closed form.
// Windows of [wt, wh, ww] tile the frames after the sink; windows are visited
// in raster order of (t, h, w) window coordinates, tokens in raster order
// inside a window, edge windows are smaller.
// ---------------------------------------------------------------------------
__global__ void window_layout_kernel(int64_t T, int64_t H, int64_t W, int64_t txt,
                                     int64_t sink_frames, int64_t wt, int64_t wh, int64_t ww,
                                     int32_t* perm, int32_t* inv) {
  const int64_t P = H * W;
  const int64_t nvid = T * P;
  const int64_t n = nvid + txt;
  const int64_t sink = sink_frames * P;
  const int64_t Tr = T - sink_frames;
  for (int64_t src = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; src < n;
       src += (int64_t)gridDim.x * blockDim.x) {
    int64_t dst = src;
    if (src >= sink && src < nvid) {
      const int64_t t = src / P - sink_frames;
      const int64_t h = (src % P) / W;
      const int64_t w = src % W;
      const int64_t t0 = (t / wt) * wt, h0 = (h / wh) * wh, w0 = (w / ww) * ww;
      const int64_t st = min(wt, Tr - t0), sh = min(wh, H - h0), sw = min(ww, W - w0);
      dst = sink + t0 * P + st * h0 * W + st * sh * w0 + ((t - t0) * sh + (h - h0)) * sw +
            (w - w0);
    }
    inv[src] = (int32_t)dst;
    perm[dst] = (int32_t)src;
  }
}

__global__ void identity_layout_kernel(int64_t n, int32_t* perm, int32_t* inv) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    perm[i] = (int32_t)i;
    inv[i] = (int32_t)i;
  }
}

// ---------------------------------------------------------------------------
// Hilbert layout.  Index of a point on the 2^bits cube, after J. Skilling,
// "Programming the Hilbert curve" (AIP Conf. Proc. 707, 2004): undo the
// excess work bit plane by bit plane (invert or exchange low bits against
// axis 0), Gray-encode across axes, then interleave the bit planes with the
// first axis most significant.
// ---------------------------------------------------------------------------
__device__ uint32_t hilbert3(uint32_t a0, uint32_t a1, uint32_t a2, int bits) {
  uint32_t x[3] = {a0, a1, a2};
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t p = q - 1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (x[i] & q) {
        x[0] ^= p;
      } else {
        const uint32_t t = (x[0] ^ x[i]) & p;
        x[0] ^= t;
        x[i] ^= t;
      }
    }
  }
  x[1] ^= x[0];
  x[2] ^= x[1];
  uint32_t t = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (x[2] & q) t ^= q - 1;
#pragma unroll
  for (int i = 0; i < 3; ++i) x[i] ^= t;
  uint32_t idx = 0;
  for (int b = bits - 1; b >= 0; --b)
#pragma unroll
    for (int i = 0; i < 3; ++i) idx = (idx << 1) | ((x[i] >> b) & 1u);
  return idx;
}

// Pass 1: key of every reordered token into inv[], presence bit into bitmap.
__global__ void hilbert_mark_kernel(int64_t T, int64_t H, int64_t W, int64_t sink_frames,
                                    int bits, uint32_t* bitmap, int32_t* inv) {
  const int64_t P = H * W;
  const int64_t sink = sink_frames * P;
  const int64_t nbody = (T - sink_frames) * P;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbody;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t t = (uint32_t)(i / P), h = (uint32_t)((i % P) / W), w = (uint32_t)(i % W);
    const uint32_t key = hilbert3(t, h, w, bits);
    inv[sink + i] = (int32_t)key;
    atomicOr(&bitmap[key >> 5], 1u << (key & 31));
  }
}

// Pass 2 (one CTA): exclusive prefix of the bitmap's popcounts.
__global__ void __launch_bounds__(1024) bitmap_prefix_kernel(const uint32_t* bitmap,
                                                             int64_t nwords, uint32_t* prefix) {
  __shared__ uint32_t part[1024];
  const int64_t per = (nwords + blockDim.x - 1) / blockDim.x;
  const int64_t beg = threadIdx.x * per;
  const int64_t end = min(nwords, beg + per);
  uint32_t s = 0;
  for (int64_t i = beg; i < end; ++i) s += __popc(bitmap[i]);
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    uint32_t v = threadIdx.x >= (unsigned)off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t run = part[threadIdx.x] - s;
  for (int64_t i = beg; i < end; ++i) {
    prefix[i] = run;
    run += __popc(bitmap[i]);
  }
}

// Pass 3: rank of each key among the present keys = its output position.
__global__ void hilbert_place_kernel(int64_t T, int64_t H, int64_t W, int64_t txt,
                                     int64_t sink_frames, const uint32_t* bitmap,
                                     const uint32_t* prefix, int32_t* perm, int32_t* inv) {
  const int64_t P = H * W;
  const int64_t sink = sink_frames * P;
  const int64_t nvid = T * P;
  const int64_t n = nvid + txt;
  for (int64_t src = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; src < n;
       src += (int64_t)gridDim.x * blockDim.x) {
    int64_t dst = src;
    if (src >= sink && src < nvid) {
      const uint32_t key = (uint32_t)inv[src];
      const uint32_t word = key >> 5, bit = key & 31;
      dst = sink + prefix[word] + __popc(bitmap[word] & ((1u << bit) - 1u));
    }
    inv[src] = (int32_t)dst;
    perm[dst] = (int32_t)src;
  }
}

int hilbert_bits_for(const sa_layout_desc& d) {
  const int64_t m = max(max(d.T - d.sink_frames, d.H), d.W);
  int b = 1;
  while ((int64_t(1) << b) < m) ++b;
  return b;
}

// ---------------------------------------------------------------------------
// Reorder: one 16-byte chunk per thread iteration, every row split into
// row_bytes/16 chunks; consecutive threads read consecutive chunks of one
// row (full 128-byte lines), rows picked through perm.  Each thread keeps
// UNROLL independent chunk copies in flight.
// ---------------------------------------------------------------------------
template <int UNROLL>
__global__ void __launch_bounds__(256) reorder_vec_kernel(const int32_t* __restrict__ perm, int64_t pstride,
                                                          const uint4* __restrict__ src,
                                                          uint4* __restrict__ dst, int64_t outer,
                                                          int64_t N, int64_t cpr, bool scatter) {
  const int64_t total = outer * N * cpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; base < total;
       base += stride * UNROLL) {
    uint4 v[UNROLL];
    int64_t out_off[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t i = base + u * stride;
      out_off[u] = -1;
      if (i < total) {
        const int64_t c = i % cpr;
        const int64_t row = i / cpr;
        const int64_t n = row % N;
        const int64_t o = row / N;
        const int64_t pn = __ldg(perm + o * pstride + n);
        const int64_t s_row = scatter ? row : o * N + pn;
        const int64_t d_row = scatter ? o * N + pn : row;
        v[u] = __ldg(src + s_row * cpr + c);
        out_off[u] = d_row * cpr + c;
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
      if (out_off[u] >= 0) __stcs(dst + out_off[u], v[u]);
  }
}

// Rows of 16 * 2^cpr_shift bytes: one CTA moves STEPS * (256 >> cpr_shift)
// consecutive rows n of one outer index o (blockIdx.y), chunk c of row rr of
// a step in thread rr * cpr + c, so a warp copies whole 128-byte lines and no
// index needs a division.  All STEPS loads of a thread are issued before
// its first store.
template <int STEPS>
__global__ void __launch_bounds__(256) reorder_rows_kernel(const int32_t* __restrict__ perm, int64_t pstride,
                                                           const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst, int64_t N, int cpr_shift,
                                                           bool scatter) {
  const int64_t o = blockIdx.y;
  const int rows_per_step = 256 >> cpr_shift;
  const int64_t n0 = (int64_t)blockIdx.x * rows_per_step * STEPS;
  const int64_t cpr = (int64_t)1 << cpr_shift;
  const int c = threadIdx.x & ((1 << cpr_shift) - 1);
  const int rr = threadIdx.x >> cpr_shift;
  const int32_t* po = perm + o * pstride;
  int64_t soff[STEPS], doff[STEPS];
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    const int64_t n = n0 + u * rows_per_step + rr;
    soff[u] = doff[u] = -1;
    if (n < N) {
      const int64_t pn = __ldg(po + n);
      soff[u] = (o * N + (scatter ? n : pn)) * cpr + c;
      doff[u] = (o * N + (scatter ? pn : n)) * cpr + c;
    }
  }
  uint4 v[STEPS];
#pragma unroll
  for (int u = 0; u < STEPS; ++u) v[u] = soff[u] >= 0 ? __ldg(src + soff[u]) : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int u = 0; u < STEPS; ++u)
    if (doff[u] >= 0) __stcs(dst + doff[u], v[u]);
}

__global__ void reorder_word_kernel(const int32_t* __restrict__ perm, int64_t pstride,
                                    const uint32_t* __restrict__ src,
                                    uint32_t* __restrict__ dst, int64_t outer, int64_t N,
                                    int64_t wpr, bool scatter) {
  const int64_t total = outer * N * wpr;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % wpr;
    const int64_t row = i / wpr;
    const int64_t n = row % N;
    const int64_t o = row / N;
    const int64_t pn = __ldg(perm + o * pstride + n);
    const int64_t s_row = scatter ? row : o * N + pn;
    const int64_t d_row = scatter ? o * N + pn : row;
    dst[d_row * wpr + c] = __ldg(src + s_row * wpr + c);
  }
}

__global__ void reorder_half_kernel(const int32_t* __restrict__ perm, int64_t pstride,
                                    const uint16_t* __restrict__ src,
                                    uint16_t* __restrict__ dst, int64_t outer, int64_t N,
                                    int64_t hpr, bool scatter) {
  const int64_t total = outer * N * hpr;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % hpr;
    const int64_t row = i / hpr;
    const int64_t n = row % N;
    const int64_t o = row / N;
    const int64_t pn = __ldg(perm + o * pstride + n);
    const int64_t s_row = scatter ? row : o * N + pn;
    const int64_t d_row = scatter ? o * N + pn : row;
    dst[d_row * hpr + c] = __ldg(src + s_row * hpr + c);
  }
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sms * 8;
  return (int)max64(1, min(want, cap));
}

}  // namespace

size_t layout_ws_bytes(const sa_layout_desc& d) {
  if (d.mode != SA_ORDER_HILBERT) return 0;
  const int bits = hilbert_bits_for(d);
  const size_t nwords = ((size_t)1 << (3 * bits)) / 32 + 1;
  return align_up(nwords * 4, 256) * 2;
}

sa_status launch_layout(const sa_layout_desc& d, int32_t* perm, int32_t* inv, void* ws,
                        cudaStream_t st) {
  const int64_t n = d.T * d.H * d.W + d.txt_len;
  const int threads = 256;
  if (d.mode == SA_ORDER_IDENTITY) {
    identity_layout_kernel<<<grid_for(n, threads), threads, 0, st>>>(n, perm, inv);
    return check_launch("identity_layout_kernel");
  }
  if (d.mode == SA_ORDER_WINDOW) {
    window_layout_kernel<<<grid_for(n, threads), threads, 0, st>>>(
        d.T, d.H, d.W, d.txt_len, d.sink_frames, d.win[0], d.win[1], d.win[2], perm, inv);
    return check_launch("window_layout_kernel");
  }
  const int bits = hilbert_bits_for(d);
  const size_t nwords = ((size_t)1 << (3 * bits)) / 32 + 1;
  uint32_t* bitmap = static_cast<uint32_t*>(ws);
  uint32_t* prefix = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + align_up(nwords * 4, 256));
  if (cudaMemsetAsync(bitmap, 0, nwords * 4, st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync failed in sa_layout_build");
  const int64_t nbody = (d.T - d.sink_frames) * d.H * d.W;
  if (nbody > 0) {
    hilbert_mark_kernel<<<grid_for(nbody, threads), threads, 0, st>>>(
        d.T, d.H, d.W, d.sink_frames, bits, bitmap, inv);
    if (sa_status e = check_launch("hilbert_mark_kernel")) return e;
    bitmap_prefix_kernel<<<1, 1024, 0, st>>>(bitmap, (int64_t)nwords, prefix);
    if (sa_status e = check_launch("bitmap_prefix_kernel")) return e;
  }
  hilbert_place_kernel<<<grid_for(n, threads), threads, 0, st>>>(
      d.T, d.H, d.W, d.txt_len, d.sink_frames, bitmap, prefix, perm, inv);
  return check_launch("hilbert_place_kernel");
}

sa_status launch_reorder(const int32_t* perm, const void* src, void* dst, int64_t outer,
                         int64_t N, int64_t row_bytes, bool scatter, cudaStream_t st, int64_t pstride) {
  const int threads = 256;
  const bool aligned16 = ((uintptr_t)src % 16 == 0) && ((uintptr_t)dst % 16 == 0);
  if (row_bytes % 16 == 0 && aligned16) {
    const int64_t cpr = row_bytes / 16;
    int shift = 0;
    while (((int64_t)1 << shift) < cpr) ++shift;
    if (((int64_t)1 << shift) == cpr && cpr <= 256 && outer <= 65535) {
      constexpr int STEPS = 4;
      const int64_t rows_per_cta = (256 >> shift) * STEPS;
      dim3 grid((unsigned)ceil_div(N, rows_per_cta), (unsigned)outer);
      reorder_rows_kernel<STEPS><<<grid, threads, 0, st>>>(perm, pstride, static_cast<const uint4*>(src),
                                                            static_cast<uint4*>(dst), N, shift, scatter);
      return check_launch("reorder_rows_kernel");
    }
    const int64_t total = outer * N * cpr;
    constexpr int U = 4;
    reorder_vec_kernel<U><<<grid_for(ceil_div(total, U), threads), threads, 0, st>>>(
        perm, pstride, static_cast<const uint4*>(src), static_cast<uint4*>(dst), outer, N, cpr, scatter);
    return check_launch("reorder_vec_kernel");
  }
  if (row_bytes % 4 == 0 && (uintptr_t)src % 4 == 0 && (uintptr_t)dst % 4 == 0) {
    const int64_t wpr = row_bytes / 4;
    reorder_word_kernel<<<grid_for(outer * N * wpr, threads), threads, 0, st>>>(
        perm, pstride, static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), outer, N, wpr,
        scatter);
    return check_launch("reorder_word_kernel");
  }
  const int64_t hpr = row_bytes / 2;
  reorder_half_kernel<<<grid_for(outer * N * hpr, threads), threads, 0, st>>>(
      perm, pstride, static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), outer, N, hpr,
      scatter);
  return check_launch("reorder_half_kernel");
}

}  // namespace sa
