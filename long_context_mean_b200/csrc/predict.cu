// Mask prediction: block pooling with the intra-block similarity guard, the
// compressed softmax with TopCdf selection, forced rows/columns, and the
// compaction of the block mask into CSR lists and a work order.
//
// [P3] SpargeAttention notes, 2.2 "selective token compression": block means
// q_hat, k_hat; a block-similarity guard theta; S_hat = q_hat k_hat^T with
// low-similarity key columns at -inf, softmax, TopCdf(tau) per row; rows of
// low-similarity query blocks and columns of low-similarity key blocks
// forced to 1.  [P2] MindIE-SD "稀疏": first-frame sink forced into full
// attention; text tokens.  [P4]/[P5]: local window and anchor keys.
//
// Readings: the similarity is the mean pairwise cosine of the block's tokens
// (diagonal included), which equals |sum_i x_i/|x_i||^2 / n^2 and is computed
// in one pass; S_hat carries 1/sqrt(d); TopCdf keeps an entry iff the mass
// sorted before it is < tau * total (ties: lower block index first); a row
// with no eligible entry selects nothing; causal: key block kb is future for
// query block qb iff kb*bk > last row of qb.
#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr int kPoolThreads = 128;
constexpr int kPoolWarps = kPoolThreads / 32;

// ---------------------------------------------------------------------------
// a2: one CTA per (head, block): block mean and mean pairwise cosine.  A warp
// covers 32/chunks tokens per step (chunks = 16-byte pieces of a token),
// four steps in flight; token norms reduce inside each token's lane group.
// With perm, token n of the block is read from row perm[n] of x and also
// written to row n of y (a1 fused with a2: the reordered copy is produced by
// the same pass that pools it).  QF = 1 + SA_Q_INT8 or 1 + SA_Q_E4M3 (bf16
// input): instead of the copy, the pass writes the block's 8-bit codes to
// row n of y8 and its scale (absmax / 127 or / 448) to qscale, reading the
// block a second time (from L2) once its absmax is known.
// ---------------------------------------------------------------------------
template <typename T, int QF = 0>
__global__ void __launch_bounds__(kPoolThreads) pool_cossim_kernel(
    const T* __restrict__ x, int64_t N, int d, int b, int nB, float* __restrict__ mean_out,
    float* __restrict__ s_out, const int32_t* __restrict__ perm, T* __restrict__ y, int32_t* status,
    uint2* __restrict__ y8 = nullptr, float* __restrict__ qscale = nullptr) {
  constexpr int EPL = 16 / sizeof(T);
  const int blk = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int64_t t0 = (int64_t)blk * b;
  const int cnt = (int)min64(b, N - t0);
  const int chunks = d / EPL;
  const int tpw = 32 / chunks;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / chunks, c = lane % chunks;
  float ax[EPL], au[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) ax[e] = au[e] = 0.f;
  float amax = 0.f;                        // QF: block absmax
  const uint4* xbh = reinterpret_cast<const uint4*>(x + bh * N * (int64_t)d);
  uint4* ybh = y ? reinterpret_cast<uint4*>(y + bh * N * (int64_t)d) : nullptr;
  const int step = kPoolWarps * tpw;
  constexpr int kInFlight = 4;
  for (int tb = warp * tpw; tb < cnt; tb += kInFlight * step) {
    uint4 raw[kInFlight];
    bool ok[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int tok = tb + u * step + sub;
      const int64_t n = t0 + tok;
      ok[u] = tok < cnt;
      int64_t src = n;
      if (perm && ok[u]) {
        src = __ldg(perm + n);
        if ((uint64_t)src >= (uint64_t)N) {   // not a permutation of [0, N)
          raise_status(status, SA_ERR_INVALID_ARG);
          ok[u] = false;
        }
      }
      raw[u] = ok[u] ? __ldg(xbh + src * chunks + c) : make_uint4(0, 0, 0, 0);
      if (ybh && ok[u]) __stcs(ybh + n * chunks + c, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      float v[EPL];
      unpack16(raw[u], T(), v);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) ss = fmaf(v[e], v[e], ss);
      for (int off = chunks >> 1; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = (ok[u] && ss > 0.f) ? 1.0f / sqrtf(ss) : 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        ax[e] += v[e];
        au[e] = fmaf(v[e], inv, au[e]);
      }
      if constexpr (QF != 0) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(v[e]));
      }
    }
  }
  for (int off = chunks; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      ax[e] += __shfl_xor_sync(0xffffffffu, ax[e], off);
      au[e] += __shfl_xor_sync(0xffffffffu, au[e], off);
    }
  }
  __shared__ float sx[kPoolWarps][256];
  __shared__ float su[kPoolWarps][256];
  __shared__ float red[kPoolWarps];
  if (lane < chunks) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sx[warp][c * EPL + e] = ax[e];
      su[warp][c * EPL + e] = au[e];
    }
  }
  __syncthreads();
  float part = 0.f;
  for (int i = threadIdx.x; i < d; i += kPoolThreads) {
    float X = 0.f, U = 0.f;
#pragma unroll
    for (int w = 0; w < kPoolWarps; ++w) {
      X += sx[w][i];
      U += su[w][i];
    }
    mean_out[(bh * nB + blk) * (int64_t)d + i] = X / (float)cnt;
    part = fmaf(U, U, part);
  }
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if (lane == 0) red[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < kPoolWarps; ++w) tot += red[w];
    s_out[bh * nB + blk] = tot / ((float)cnt * (float)cnt);
  }
  if constexpr (QF != 0) {
    static_assert(sizeof(T) == 2, "8-bit codes are written from bf16 input");
    constexpr int FMT = QF - 1;
    __shared__ float wmax[kPoolWarps];
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) wmax[warp] = amax;
    __syncthreads();
    float A = 0.f;
#pragma unroll
    for (int w = 0; w < kPoolWarps; ++w) A = fmaxf(A, wmax[w]);
    const float qmax = FMT == SA_Q_E4M3 ? 448.0f : 127.0f;
    const float qinv = A > 0.f ? __fdiv_rn(qmax, A) : 0.f;
    if (threadIdx.x == 0) qscale[bh * nB + blk] = A > 0.f ? __fdiv_rn(A, qmax) : 0.f;
    uint2* y8bh = y8 + bh * N * (int64_t)chunks;
    for (int tb = warp * tpw; tb < cnt; tb += step) {
      const int tok = tb + sub;
      if (tok >= cnt) continue;
      const int64_t n = t0 + tok;
      const int64_t src = perm ? (int64_t)__ldg(perm + n) : n;
      if ((uint64_t)src >= (uint64_t)N) continue;          // raised in the first pass
      y8bh[n * chunks + c] = quant8<FMT>(__ldg(xbh + src * chunks + c), qinv);
    }
  }
}

// ---------------------------------------------------------------------------
// Shared row rules (structure-forced rows/columns, window, causal validity).
// ---------------------------------------------------------------------------
struct RowRules {
  int64_t N, sink, txt, window, anchor;
  int bq, bk, causal;
  __device__ bool struct_row(int64_t qb) const {
    const int64_t i0 = qb * bq, i1 = min(N, (qb + 1) * bq);
    return i0 < sink || (txt > 0 && i1 - 1 >= N - txt);
  }
  __device__ bool struct_col(int64_t kb) const {
    const int64_t j0 = kb * bk, j1 = min(N, (kb + 1) * bk);
    return j0 < sink || j0 < anchor || (txt > 0 && j1 - 1 >= N - txt);
  }
  __device__ bool in_window(int64_t qb, int64_t kb) const {
    if (window <= 0) return false;
    const int64_t i0 = qb * bq, i1 = min(N, (qb + 1) * bq);
    const int64_t j0 = kb * bk, j1 = min(N, (kb + 1) * bk);
    return (i1 - 1 >= j0) && (i0 - (j1 - 1) < window);
  }
  __device__ bool valid(int64_t qb, int64_t kb) const {
    if (!causal) return true;
    return kb * bk <= min(N, (qb + 1) * bq) - 1;
  }
};

constexpr int kRowThreads = 256;

__device__ __forceinline__ int block_reduce_sum_int(int v, int* sh) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int r = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += sh[w];
  return r;
}

__device__ __forceinline__ int block_reduce_min_int(int v, int* sh) {
  for (int off = 16; off > 0; off >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int r = 0x7fffffff;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = min(r, sh[w]);
  return r;
}

// Finishes one mask row: writes the bytes, the row count, and raises
// SA_ERR_EMPTY_ROW when the block's first query row would see no key
// (causal: some kept kb with kb*bk <= first row; else any kept kb).
__device__ void finish_row(const uint8_t* flags, int64_t u, int64_t qb, int64_t nkb,
                           const RowRules& r, uint8_t* mask_row_out, int32_t* counts,
                           int32_t* status, int* sh_int) {
  int cnt = 0, first = 0x7fffffff;
  for (int64_t kb = threadIdx.x; kb < nkb; kb += blockDim.x) {
    const uint8_t f = flags[kb];
    mask_row_out[kb] = f;
    if (f) {
      ++cnt;
      first = min(first, (int)kb);
    }
  }
  cnt = block_reduce_sum_int(cnt, sh_int);
  first = block_reduce_min_int(first, sh_int);
  if (threadIdx.x == 0) {
    counts[u] = cnt;
    const bool empty = r.causal ? (cnt == 0 || (int64_t)first * r.bk > qb * r.bq) : cnt == 0;
    if (empty) raise_status(status, SA_ERR_EMPTY_ROW);
  }
}

// ---------------------------------------------------------------------------
// a3 + a4: one CTA per (head, group of G <= 8 query blocks).  Scores: thread
// i takes the key blocks kb = i, i + 256, ... and computes q_hat[r] . k_hat[kb]
// for every row r of the group, reading its k_hat row from global memory
// (L2-resident, each element read once per group) and the q_hat rows from
// shared memory (the same address in every lane: broadcast), so the loop is
// bound by the FMA pipe.  Then warp r alone finishes row r: softmax and
// TopCdf (an arg-max loop over register-resident keys when the row is short
// and few blocks are picked, else a bisection for the last kept
// probability), the union with the forced parts and the causal AND -- with
// warp-level synchronisation only.
// Dynamic shared memory: q_hat [8][d] | scores [G][nkb rounded to 4] (fp32;
// the bisection turns a row's scores into its probabilities in place, the
// padding holding zeros) | flags [G][nkb rounded to 16] (u8).
// ---------------------------------------------------------------------------
constexpr int kMaxRowsPerCta = 8;
constexpr int kFastKeys = 16;     // keys per lane on the fast TopCdf path (nkb <= 512)
constexpr int kFastPicks = 128;   // picks before the fast path defers to the sort

int score_rows_per_cta(int P2) {
  int g = 65536 / (P2 * 4);
  return g < 1 ? 1 : (g > kMaxRowsPerCta ? kMaxRowsPerCta : g);
}

size_t score_smem_bytes(int d, int64_t nkb, int P2, int G) {
  (void)P2;
  const size_t nkb16 = (size_t)((nkb + 15) / 16) * 16;
  const size_t nkb4 = (size_t)((nkb + 3) / 4) * 4;
  return (size_t)kMaxRowsPerCta * d * 4 + (size_t)G * nkb4 * 4 + (size_t)G * nkb16;
}

__device__ __forceinline__ float warp_max(float v) {
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__global__ void __launch_bounds__(kRowThreads) score_topcdf_kernel(
    const float* __restrict__ qhat, const float* __restrict__ khat, const float* __restrict__ sq,
    const float* __restrict__ sk, int64_t Hq, int64_t Hkv, int64_t nqb, int64_t nkb, int d,
    int P2, int G, float tau, float theta, RowRules rules, uint8_t* __restrict__ mask,
    int32_t* __restrict__ counts, int32_t* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nkb16 = (int)((nkb + 15) / 16) * 16;
  const int nkb4 = (int)((nkb + 3) / 4) * 4;   // score row stride: float4-aligned rows
  float* qs = reinterpret_cast<float*>(smem);
  float* sc = reinterpret_cast<float*>(smem + (size_t)kMaxRowsPerCta * d * 4);
  uint8_t* flags = reinterpret_cast<uint8_t*>(sc + G * nkb4);
  __shared__ int s_forced[kMaxRowsPerCta];

  const int64_t bh = blockIdx.y;
  const int64_t qb0 = (int64_t)blockIdx.x * G;
  const int rows = (int)min64(G, nqb - qb0);
  const int64_t b = bh / Hq, h = bh % Hq;
  const int64_t g = b * Hkv + h / (Hq / Hkv);
  const bool guard = theta > 0.f;
  const float scale = rsqrtf((float)d);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < kMaxRowsPerCta) {
    const int r = threadIdx.x;
    const int64_t u = bh * nqb + qb0 + r;
    s_forced[r] = (r >= rows) ? 1 : ((rules.struct_row(qb0 + r) || (guard && sq[u] < theta)) ? 1 : 0);
  }
  for (int i = threadIdx.x; i < rows * d; i += blockDim.x) qs[i] = qhat[(bh * nqb + qb0) * (int64_t)d + i];
  __syncthreads();
  int any_scored = 0;
  for (int r = 0; r < rows; ++r) any_scored |= !s_forced[r];

  if (any_scored) {
    const float4* kg4 = reinterpret_cast<const float4*>(khat + g * nkb * (int64_t)d);
    const float4* qs4 = reinterpret_cast<const float4*>(qs);
    const int nf4 = d / 4;
    for (int64_t kb = threadIdx.x; kb < nkb; kb += kRowThreads) {
      uint32_t need = 0;   // rows of the group that score this key block
      const bool col_ok = !(guard && sk[g * nkb + kb] < theta);
#pragma unroll
      for (int r = 0; r < kMaxRowsPerCta; ++r)
        if (r < rows && col_ok && !s_forced[r] && rules.valid(qb0 + r, kb)) need |= 1u << r;
      float a[kMaxRowsPerCta][4];
#pragma unroll
      for (int r = 0; r < kMaxRowsPerCta; ++r) a[r][0] = a[r][1] = a[r][2] = a[r][3] = 0.f;
      if (need) {
        const float4* kr = kg4 + kb * nf4;
        for (int e = 0; e < nf4; ++e) {
          const float4 y = __ldg(kr + e);
#pragma unroll
          for (int r = 0; r < kMaxRowsPerCta; ++r) {
            if (r < rows) {
              const float4 x = qs4[r * nf4 + e];
              a[r][0] = fmaf(x.x, y.x, a[r][0]);
              a[r][1] = fmaf(x.y, y.y, a[r][1]);
              a[r][2] = fmaf(x.z, y.z, a[r][2]);
              a[r][3] = fmaf(x.w, y.w, a[r][3]);
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kMaxRowsPerCta; ++r)
        if (r < rows) sc[r * nkb4 + kb] = ((need >> r) & 1u) ? ((a[r][0] + a[r][1]) + (a[r][2] + a[r][3])) * scale
                                                              : -INFINITY;
    }
    __syncthreads();
  }

  if (warp >= rows) return;
  // ---- warp `warp` finishes row r = warp ----
  const int r = warp;
  const int64_t qb = qb0 + r;
  const int64_t u = bh * nqb + qb;
  const bool row_forced = s_forced[r] != 0;
  float* pr = sc + (size_t)r * nkb4;   // probabilities replace the scores (bisection)
  uint8_t* fl = flags + (size_t)r * nkb16;
  for (int64_t kb = lane; kb < nkb; kb += 32) fl[kb] = 0;
  if (!row_forced) {
    const float* srow = sc + r * nkb4;
    float mx = -INFINITY;
    for (int64_t kb = lane; kb < nkb; kb += 32) mx = fmaxf(mx, srow[kb]);
    mx = warp_max(mx);
    bool done = false;
    if (mx > -INFINITY && P2 <= 32 * kFastKeys) {
      // Fast path: repeated warp-wide arg-max over register-resident keys,
      // accumulating the mass in sorted order; TopCdf usually stops after a
      // few picks.  Gives up after kFastPicks picks (the bisection below then
      // decides the row from scratch).
      uint64_t key[kFastKeys];
      float part = 0.f;
#pragma unroll
      for (int q = 0; q < kFastKeys; ++q) {
        const int kb = lane + 32 * q;
        key[q] = 0ull;
        if (kb < nkb) {
          const float sv = srow[kb];
          const float pv = (sv == -INFINITY) ? 0.f : expf(sv - mx);
          key[q] = ((uint64_t)__float_as_uint(pv) << 32) | (uint32_t)(~(uint32_t)kb);
          part += pv;
        }
      }
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const float limit = tau * part;
      float cum = 0.f;
      for (int pick = 0; pick < kFastPicks; ++pick) {
        uint64_t best = 0ull;
#pragma unroll
        for (int q = 0; q < kFastKeys; ++q) best = key[q] > best ? key[q] : best;
        for (int off = 16; off > 0; off >>= 1) {
          const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
          best = o > best ? o : best;
        }
        const float pv = __uint_as_float((uint32_t)(best >> 32));
        if (!(pv > 0.f) || !(cum < limit)) {
          done = true;
          break;
        }
        const uint32_t kb = ~(uint32_t)best;
        if ((int)(kb & 31) == lane) fl[kb] = 1;
        // Keys are unique (the block index is part of the key): clearing by
        // value needs no computed index, so key[] stays in registers.
#pragma unroll
        for (int q = 0; q < kFastKeys; ++q) key[q] = key[q] == best ? 0ull : key[q];
        cum += pv;
      }
      if (!done) {
        for (int64_t kb = lane; kb < nkb; kb += 32) fl[kb] = 0;
      }
      __syncwarp();
    }
    if (mx > -INFINITY && !done) {
      // Threshold search for rows the fast path does not settle.  With p
      // sorted descending (ties by index), block j is kept iff the mass
      // sorted before it is < tau * total.  Let f(t) be the mass of the p
      // whose bit pattern exceeds t (p >= 0: bit order = value order); f
      // falls as t rises.  The smallest t* with f(t*) < tau * total is the
      // bit pattern of the last value kept: every p above it is kept, and the
      // blocks whose p equals it are kept in index order while f(t*) + r p <
      // tau * total (r = rank among them).  t* is found by bisection over the
      // bit patterns of (0, 1] (p = exp(s - max) <= 1).
      for (int kb = lane; kb < nkb4; kb += 32) {
        const float sv = kb < nkb ? srow[kb] : -INFINITY;
        pr[kb] = (sv == -INFINITY) ? 0.f : expf(sv - mx);
      }
      __syncwarp();
      const float4* pr4 = reinterpret_cast<const float4*>(pr);
      auto mass_above = [&](uint32_t t) -> float {
        float m0 = 0.f, m1 = 0.f;
        for (int q = lane; q < nkb4 / 4; q += 32) {
          const float4 v = pr4[q];
          m0 += (__float_as_uint(v.x) > t ? v.x : 0.f) + (__float_as_uint(v.y) > t ? v.y : 0.f);
          m1 += (__float_as_uint(v.z) > t ? v.z : 0.f) + (__float_as_uint(v.w) > t ? v.w : 0.f);
        }
        float m = m0 + m1;
        for (int off = 16; off > 0; off >>= 1) m += __shfl_xor_sync(0xffffffffu, m, off);
        return m;
      };
      const float limit = tau * mass_above(0u);
      uint32_t lo = 0u, hi = 0x3F800000u;   // f(lo) >= limit (tau <= 1), f(hi) = 0 < limit
      while (hi - lo > 1u) {
        const uint32_t mid = lo + (hi - lo) / 2u;
        if (mass_above(mid) < limit) hi = mid;
        else lo = mid;
      }
      const float above = mass_above(hi);
      const float vstar = __uint_as_float(hi);
      uint32_t run = 0;
      for (int64_t kb0 = 0; kb0 < nkb; kb0 += 32) {
        const int64_t kb = kb0 + lane;
        const uint32_t bits = kb < nkb ? __float_as_uint(pr[kb]) : 0u;
        const bool tie = kb < nkb && bits == hi;
        const unsigned bal = __ballot_sync(0xffffffffu, tie);
        bool keep = kb < nkb && bits > hi;
        if (tie) keep = above + (float)(run + __popc(bal & ((1u << lane) - 1u))) * vstar < limit;
        if (keep) fl[kb] = 1;
        run += __popc(bal);
      }
    }
  }
  __syncwarp();
  int cnt = 0, first = 0x7fffffff;
  uint8_t* mrow = mask + u * nkb;
  for (int64_t kb = lane; kb < nkb; kb += 32) {
    const bool col = rules.struct_col(kb) || (guard && sk[g * nkb + kb] < theta);
    const bool keep = rules.valid(qb, kb) && (row_forced || fl[kb] || col || rules.in_window(qb, kb));
    mrow[kb] = keep ? 1 : 0;
    if (keep) {
      ++cnt;
      first = min(first, (int)kb);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    first = min(first, __shfl_xor_sync(0xffffffffu, first, off));
  }
  if (lane == 0) {
    counts[u] = cnt;
    const bool empty = rules.causal ? (cnt == 0 || (int64_t)first * rules.bk > qb * rules.bq) : cnt == 0;
    if (empty) raise_status(status, SA_ERR_EMPTY_ROW);
  }
}

// A caller-supplied mask row: AND causal validity, copy, count, check.
__global__ void __launch_bounds__(kRowThreads) mask_copy_kernel(
    const uint8_t* __restrict__ in, int64_t nqb, int64_t nkb, RowRules rules,
    uint8_t* __restrict__ out, int32_t* __restrict__ counts, int32_t* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint8_t* flags = smem;
  __shared__ int shi[32];
  const int64_t u = blockIdx.x;
  const int64_t qb = u % nqb;
  for (int64_t kb = threadIdx.x; kb < nkb; kb += blockDim.x)
    flags[kb] = (in[u * nkb + kb] != 0 && rules.valid(qb, kb)) ? 1 : 0;
  __syncthreads();
  finish_row(flags, u, qb, nkb, rules, out + u * nkb, counts, status, shi);
}

// ---------------------------------------------------------------------------
// CSR: one CTA scans the row counts into row_ptr and checks capacity.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) rows_scan_kernel(const int32_t* __restrict__ counts,
                                                         int64_t R, int64_t capacity,
                                                         int32_t* __restrict__ row_ptr,
                                                         int64_t* kept_total, int32_t* status) {
  __shared__ int64_t part[1024];
  const int64_t per = (R + blockDim.x - 1) / blockDim.x;
  const int64_t beg = threadIdx.x * per, end = min(R, beg + per);
  int64_t s = 0;
  for (int64_t i = beg; i < end; ++i) s += counts[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    const int64_t v = threadIdx.x >= (unsigned)off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int64_t run = part[threadIdx.x] - s;
  for (int64_t i = beg; i < end; ++i) {
    row_ptr[i] = (int32_t)min64(run, INT32_MAX);
    run += counts[i];
  }
  if (threadIdx.x == blockDim.x - 1) {
    const int64_t tot = part[blockDim.x - 1];
    row_ptr[R] = (int32_t)min64(tot, INT32_MAX);
    *kept_total = tot;
    if (tot > capacity || tot > INT32_MAX) raise_status(status, SA_ERR_CAPACITY);
  }
}

// One warp per row: ascending kept block indices by ballot compaction.
__global__ void fill_cols_kernel(const uint8_t* __restrict__ mask, int64_t R, int64_t nkb,
                                 const int32_t* __restrict__ row_ptr, int64_t capacity,
                                 int32_t* __restrict__ col_idx) {
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= R) return;
  const int64_t lo = row_ptr[warp];
  const int64_t hi = row_ptr[warp + 1];
  if (hi > capacity) return;  // capacity error already raised
  int64_t pos = lo;
  for (int64_t kb0 = 0; kb0 < nkb; kb0 += 32) {
    const int64_t kb = kb0 + lane;
    const bool f = kb < nkb && mask[warp * nkb + kb] != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    if (f) col_idx[pos + __popc(bal & ((1u << lane) - 1u))] = (int32_t)kb;
    pos += __popc(bal);
  }
}

// Work order: stable LSD radix sort of rows by key = 4095 - count (3 passes
// of 4 bits), i.e. descending count, ties by ascending row index.  One CTA;
// each thread owns a contiguous range of the current sequence and keeps its
// 16 digit counts in a padded row of shared memory (stride 17: no bank
// conflicts); the scatter offsets come from a scan in (digit, thread) order
// done with warp shuffles, which keeps the scatter stable.  When the rows
// fit (R <= kOrderSmemRows) the keys and the intermediate sequences live in
// shared memory and only the final pass writes `order`.
constexpr int kOrderThreads = 1024;
constexpr int kOrderWarps = kOrderThreads / 32;
constexpr int kOrderSmemRows = 8192;
constexpr int kHistStride = 17;

__global__ void __launch_bounds__(kOrderThreads) order_kernel(const int32_t* __restrict__ counts,
                                                              int64_t R, int32_t* __restrict__ tmp,
                                                              int32_t* __restrict__ order) {
  extern __shared__ uint32_t dyn[];
  uint32_t* hist = dyn;                                   // [kOrderThreads][17]
  const bool in_smem = R <= kOrderSmemRows;
  uint16_t* skey = reinterpret_cast<uint16_t*>(dyn + kHistStride * kOrderThreads);   // [R] key of row
  int32_t* sa = reinterpret_cast<int32_t*>(skey + (in_smem ? kOrderSmemRows : 0));   // [R] sequences
  int32_t* sb = sa + (in_smem ? kOrderSmemRows : 0);
  __shared__ uint32_t wtot[kOrderWarps][16];              // per-warp digit totals, then warp offsets
  __shared__ uint32_t dtot[16];                           // digit totals
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* my = hist + tid * kHistStride;
  const int64_t per = (R + kOrderThreads - 1) / kOrderThreads;
  const int64_t beg = tid * per, end = min(R, beg + per);
  if (in_smem) {
    for (int64_t i = tid; i < R; i += kOrderThreads) skey[i] = (uint16_t)(4095u - (uint32_t)counts[i]);
    __syncthreads();
  }
  auto key_of = [&](int32_t row) -> uint32_t {
    return in_smem ? (uint32_t)skey[row] : 4095u - (uint32_t)counts[row];
  };
  for (int pass = 0; pass < 3; ++pass) {
    // source and destination of this pass: rows in natural order first, the
    // final pass writes `order`
    const int32_t* src = pass == 0 ? nullptr : (in_smem ? (pass == 1 ? sa : sb) : (pass == 1 ? order : tmp));
    int32_t* dst = pass == 2 ? order : (in_smem ? (pass == 0 ? sa : sb) : (pass == 0 ? order : tmp));
    const int shift = 4 * pass;
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) my[dgt] = 0;
    for (int64_t i = beg; i < end; ++i) {
      const int32_t row = src ? src[i] : (int32_t)i;
      my[(key_of(row) >> shift) & 15u] += 1;
    }
    // Offsets: entry (digit, thread) starts after every entry of smaller
    // digits and after the same digit's entries of smaller threads.
    uint32_t c[16], x[16];
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) x[dgt] = c[dgt] = my[dgt];
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) {
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, x[dgt], off);
        if (lane >= off) x[dgt] += o;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int dgt = 0; dgt < 16; ++dgt) wtot[warp][dgt] = x[dgt];
    }
    __syncthreads();
    if (tid < 16) {   // thread `dgt`: exclusive scan of the warp totals of its digit
      uint32_t run = 0;
      for (int w = 0; w < kOrderWarps; ++w) {
        const uint32_t t = wtot[w][tid];
        wtot[w][tid] = run;
        run += t;
      }
      dtot[tid] = run;
    }
    __syncthreads();
    uint32_t base = 0;
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) {
      my[dgt] = base + wtot[warp][dgt] + x[dgt] - c[dgt];
      base += dtot[dgt];
    }
    __syncthreads();
    for (int64_t i = beg; i < end; ++i) {
      const int32_t row = src ? src[i] : (int32_t)i;
      uint32_t& slot = my[(key_of(row) >> shift) & 15u];
      dst[slot] = row;
      slot += 1;
    }
    __syncthreads();
  }
}

sa_status launch_lists(const sa_shape& s, int bq, int bk, int32_t* counts, int32_t* tmp,
                       sa_mask& out, cudaStream_t st) {
  const int64_t R = s.B * s.Hq * out.nqb;
  rows_scan_kernel<<<1, 1024, 0, st>>>(counts, R, out.col_capacity, out.row_ptr, out.kept_total,
                                       out.status);
  if (sa_status e = check_launch("rows_scan_kernel")) return e;
  const int64_t warps_per_block = 8;
  fill_cols_kernel<<<(unsigned)ceil_div(R, warps_per_block), 32 * warps_per_block, 0, st>>>(
      out.block_mask, R, out.nkb, out.row_ptr, out.col_capacity, out.col_idx);
  if (sa_status e = check_launch("fill_cols_kernel")) return e;
  size_t hist_bytes = (size_t)kHistStride * kOrderThreads * sizeof(uint32_t);
  if (R <= kOrderSmemRows) hist_bytes += (size_t)kOrderSmemRows * (2 + 4 + 4);   // keys + two sequences
  if (cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)hist_bytes) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(order_kernel) failed");
  order_kernel<<<1, kOrderThreads, hist_bytes, st>>>(counts, R, tmp, out.order);
  return check_launch("order_kernel");
}

RowRules make_rules(const sa_shape& s, const sa_mask_params& p) {
  RowRules r;
  r.N = s.N;
  r.sink = p.sink_tokens;
  r.txt = p.txt_len;
  r.window = p.local_window;
  r.anchor = p.anchor_tokens;
  r.bq = p.bq;
  r.bk = p.bk;
  r.causal = p.causal;
  return r;
}

template <typename T>
sa_status launch_pool(const void* x, int64_t BH, int64_t N, int d, int b, int64_t nB, float* mean,
                      float* sim, const int32_t* perm, void* y, int32_t* status, cudaStream_t st) {
  dim3 grid((unsigned)nB, (unsigned)BH);
  pool_cossim_kernel<T><<<grid, kPoolThreads, 0, st>>>(static_cast<const T*>(x), N, d, b, (int)nB,
                                                       mean, sim, perm, static_cast<T*>(y), status);
  return check_launch("pool_cossim_kernel");
}

// Pooling with 8-bit codes and block scales instead of the reordered copy.
sa_status launch_pool_codes(const void* x, int64_t BH, int64_t N, int d, int b, int64_t nB, float* mean,
                            float* sim, const int32_t* perm, int32_t fmt, void* y8, float* qscale, int32_t* status,
                            cudaStream_t st) {
  dim3 grid((unsigned)nB, (unsigned)BH);
  if (fmt == SA_Q_E4M3)
    pool_cossim_kernel<uint16_t, 1 + SA_Q_E4M3><<<grid, kPoolThreads, 0, st>>>(
        static_cast<const uint16_t*>(x), N, d, b, (int)nB, mean, sim, perm, nullptr, status,
        static_cast<uint2*>(y8), qscale);
  else
    pool_cossim_kernel<uint16_t, 1 + SA_Q_INT8><<<grid, kPoolThreads, 0, st>>>(
        static_cast<const uint16_t*>(x), N, d, b, (int)nB, mean, sim, perm, nullptr, status,
        static_cast<uint2*>(y8), qscale);
  return check_launch("pool_cossim_kernel");
}

}  // namespace

size_t predict_ws_bytes(const sa_shape& s, int bq, int bk, size_t off[6]) {
  const int64_t nqb = ceil_div(s.N, bq), nkb = ceil_div(s.N, bk);
  const int64_t R = s.B * s.Hq * nqb;
  size_t o = 0;
  const size_t sizes[6] = {(size_t)(s.B * s.Hq * nqb * s.d) * 4, (size_t)(s.B * s.Hkv * nkb * s.d) * 4,
                           (size_t)(s.B * s.Hq * nqb) * 4,      (size_t)(s.B * s.Hkv * nkb) * 4,
                           (size_t)R * 4,                        (size_t)R * 4};
  for (int i = 0; i < 6; ++i) {
    off[i] = o;
    o += align_up(sizes[i], 256);
  }
  return o;
}

PredictWs predict_ws_carve(void* ws, const sa_shape& s, int bq, int bk) {
  size_t off[6];
  predict_ws_bytes(s, bq, bk, off);
  char* p = static_cast<char*>(ws);
  PredictWs w;
  w.qhat = reinterpret_cast<float*>(p + off[0]);
  w.khat = reinterpret_cast<float*>(p + off[1]);
  w.sq = reinterpret_cast<float*>(p + off[2]);
  w.sk = reinterpret_cast<float*>(p + off[3]);
  w.counts = reinterpret_cast<int32_t*>(p + off[4]);
  w.tmp = reinterpret_cast<int32_t*>(p + off[5]);
  return w;
}

size_t lists_ws_bytes(const sa_shape& s, int bq, int) {
  const int64_t R = s.B * s.Hq * ceil_div(s.N, bq);
  return align_up((size_t)R * 4, 256) * 2;
}

sa_status launch_predict(const void* q, const void* k, const sa_shape& s,
                         const sa_mask_params& p, const PredictWs& w, sa_mask& out,
                         cudaStream_t st, const int32_t* perm, void* q_r, void* k_r, const PoolCodes* codes) {
  const int64_t nqb = out.nqb, nkb = out.nkb;
  if (cudaMemsetAsync(out.status, 0, sizeof(int32_t), st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync(status) failed");
  sa_status e;
  if (codes) {   // bf16 input: codes and scales instead of reordered copies
    if ((e = launch_pool_codes(q, s.B * s.Hq, s.N, (int)s.d, p.bq, nqb, w.qhat, w.sq, perm, codes->format,
                               codes->q8, codes->q_scales, out.status, st)))
      return e;
    if ((e = launch_pool_codes(k, s.B * s.Hkv, s.N, (int)s.d, p.bk, nkb, w.khat, w.sk, perm, codes->format,
                               codes->k8, codes->k_scales, out.status, st)))
      return e;
  } else if (s.dtype == SA_BF16) {
    if ((e = launch_pool<uint16_t>(q, s.B * s.Hq, s.N, (int)s.d, p.bq, nqb, w.qhat, w.sq, perm, q_r,
                                   out.status, st)))
      return e;
    if ((e = launch_pool<uint16_t>(k, s.B * s.Hkv, s.N, (int)s.d, p.bk, nkb, w.khat, w.sk, perm, k_r,
                                   out.status, st)))
      return e;
  } else {
    if ((e = launch_pool<float>(q, s.B * s.Hq, s.N, (int)s.d, p.bq, nqb, w.qhat, w.sq, perm, q_r,
                                out.status, st)))
      return e;
    if ((e = launch_pool<float>(k, s.B * s.Hkv, s.N, (int)s.d, p.bk, nkb, w.khat, w.sk, perm, k_r,
                                out.status, st)))
      return e;
  }
  int P2 = 1;
  while (P2 < nkb) P2 <<= 1;
  const int G = score_rows_per_cta(P2);
  const size_t smem = score_smem_bytes((int)s.d, nkb, P2, G);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(score_topcdf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(score_topcdf_kernel) failed");
  }
  dim3 grid((unsigned)ceil_div(nqb, G), (unsigned)(s.B * s.Hq));
  score_topcdf_kernel<<<grid, kRowThreads, smem, st>>>(
      w.qhat, w.khat, w.sq, w.sk, s.Hq, s.Hkv, nqb, nkb, (int)s.d, P2, G, p.tau, p.theta,
      make_rules(s, p), out.block_mask, w.counts, out.status);
  if ((e = check_launch("score_topcdf_kernel"))) return e;
  return launch_lists(s, p.bq, p.bk, w.counts, w.tmp, out, st);
}

sa_status launch_mask_from_blocks(const uint8_t* in, const sa_shape& s, int bq, int bk, int causal,
                                  int32_t* counts, int32_t* tmp, sa_mask& out, cudaStream_t st) {
  if (cudaMemsetAsync(out.status, 0, sizeof(int32_t), st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync(status) failed");
  sa_mask_params p{};
  p.bq = bq;
  p.bk = bk;
  p.causal = causal;
  const int64_t R = s.B * s.Hq * out.nqb;
  const size_t smem = align_up((size_t)out.nkb, 16);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(mask_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(mask_copy_kernel) failed");
  }
  mask_copy_kernel<<<(unsigned)R, kRowThreads, smem, st>>>(in, out.nqb, out.nkb, make_rules(s, p),
                                                          out.block_mask, counts, out.status);
  if (sa_status e = check_launch("mask_copy_kernel")) return e;
  return launch_lists(s, bq, bk, counts, tmp, out, st);
}

}  // namespace sa
