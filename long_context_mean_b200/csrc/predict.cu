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

constexpr int kPoolThreads = 256;
constexpr int kPoolWarps = kPoolThreads / 32;
constexpr int kPoolLoads = 4;   // 16-byte loads a lane has in flight

// Two fp32 values in one 64-bit register for the packed fp32x2 pipe.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// A 16-byte vector of elements as fp32 pairs (8 bf16 -> 4 pairs, 4 fp32 -> 2).
__device__ __forceinline__ void pairs16(const uint4& u, uint16_t, uint64_t* p) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}
__device__ __forceinline__ void pairs16(const uint4& u, float, uint64_t* p) {
  p[0] = f2(__uint_as_float(u.x), __uint_as_float(u.y));
  p[1] = f2(__uint_as_float(u.z), __uint_as_float(u.w));
}

// ---------------------------------------------------------------------------
// a2: block mean and mean pairwise cosine of every (head, block) unit.  Each
// warp owns whole units (unit = its global warp index, + the grid's warps,
// ...), so no barrier couples the warps and the SM keeps as many of them in
// flight as registers allow.  A token is CH lanes x 16 bytes (CH = chunks per
// token, a template parameter); a warp step covers 32 / CH tokens and a lane
// has kPoolLoads steps of loads in flight before it uses any.  The token norm
// reduces inside the token's lane group (independent shuffle chains for the
// loads in flight); Σx and Σx/‖x‖ (hardware reciprocal square root)
// accumulate on the packed fp32x2 pipe and reduce across the token groups at
// the end.  With perm, token n of the block is read from row perm[n] of x
// (the block's rows staged in the warp's shared memory first; an entry
// outside [0, N) raises SA_ERR_INVALID_ARG and the token reads as zeros and
// is not written) and also written to row n of y (a1 fused with a2: the
// reordered copy is produced by the same pass that pools it).  The block mean
// goes to mean_out[(bh * nB + blk) * d + i], or with mean_tstride > 0 to
// mean_out[(bh * d + i) * mean_tstride + blk] (transposed: one row per
// feature, blocks contiguous).  QF = 1 + SA_Q_INT8 or 1 + SA_Q_E4M3 (bf16
// input): instead of the copy, the pass writes the block's 8-bit codes to row
// n of y8 and its scale (absmax / 127 or / 448) to qscale, reading the block
// a second time (from L2) once its absmax is known.
// ---------------------------------------------------------------------------
// One pooled tensor of a launch (Q and K go through the same launch: their
// units follow one another in one persistent grid).
struct PoolJob {
  const void* x;          // [BH, N, d]
  int64_t BH;             // heads (batch x heads); 0: no job
  int b, nB;              // block size, blocks per head
  float* mean_out;        // block means, layout per mean_tstride
  int64_t mean_tstride;   // 0: [BH, nB, d]; > 0: [BH, d, mean_tstride]
  float* s_out;           // block similarities [BH, nB]
  void* y;                // reordered copy (nullable)
  uint2* y8;              // 8-bit codes (QF)
  float* qscale;          // block scales (QF)
};

template <typename T, int CH, int QF = 0>
__global__ void __launch_bounds__(kPoolThreads, 4) pool_cossim_kernel(PoolJob j0, PoolJob j1, int64_t N,
                                                                       const int32_t* __restrict__ perm,
                                                                       int32_t* status) {
  constexpr int EPL = 16 / sizeof(T);   // elements per chunk
  constexpr int NP = EPL / 2;           // fp32 pairs per chunk
  constexpr int d = CH * EPL;
  constexpr int TPW = 32 / CH;          // tokens per warp step
  static_assert(CH >= 1 && CH <= 32 && (CH & (CH - 1)) == 0, "chunks per token: a power of two <= 32");
  __shared__ int32_t srow_all[kPoolWarps][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / CH, c = lane % CH;
  int32_t* srow = srow_all[warp];
  const int64_t units0 = j0.BH * j0.nB;
  const int64_t units = units0 + j1.BH * j1.nB;
  const int64_t wstride = (int64_t)gridDim.x * kPoolWarps;
  for (int64_t gunit = (int64_t)blockIdx.x * kPoolWarps + warp; gunit < units; gunit += wstride) {
    const bool second = gunit >= units0;
    const int64_t unit = second ? gunit - units0 : gunit;
    const T* __restrict__ x = static_cast<const T*>(second ? j1.x : j0.x);
    const int b = second ? j1.b : j0.b;
    const int nB = second ? j1.nB : j0.nB;
    float* __restrict__ mean_out = second ? j1.mean_out : j0.mean_out;
    const int64_t mean_tstride = second ? j1.mean_tstride : j0.mean_tstride;
    float* __restrict__ s_out = second ? j1.s_out : j0.s_out;
    T* __restrict__ y = static_cast<T*>(second ? j1.y : j0.y);
    uint2* __restrict__ y8 = second ? j1.y8 : j0.y8;
    float* __restrict__ qscale = second ? j1.qscale : j0.qscale;
    const int64_t bh = unit / nB;
    const int blk = (int)(unit - bh * nB);
    const int64_t t0 = (int64_t)blk * b;
    const int cnt = (int)min64(b, N - t0);
    const uint4* xbh = reinterpret_cast<const uint4*>(x + bh * N * (int64_t)d) + c;
    uint4* ybh = y ? reinterpret_cast<uint4*>(y + bh * N * (int64_t)d) + t0 * CH + c : nullptr;
    if (perm) {
      __syncwarp();   // the previous unit's rows are no longer read
      for (int i = lane; i < cnt; i += 32) {
        const int32_t s = __ldg(perm + t0 + i);
        if ((uint32_t)s >= (uint64_t)N) raise_status(status, SA_ERR_INVALID_ARG);   // not a permutation of [0, N)
        srow[i] = (uint32_t)s < (uint64_t)N ? s : -1;
      }
      __syncwarp();
    }
    uint64_t ax[NP], au[NP];
#pragma unroll
    for (int e = 0; e < NP; ++e) ax[e] = au[e] = f2(0.f, 0.f);
    float amax = 0.f;
    for (int tb = 0; tb < cnt; tb += kPoolLoads * TPW) {   // uniform: the shuffles need every lane
      uint4 raw[kPoolLoads];
      uint32_t okm = 0;
#pragma unroll
      for (int u = 0; u < kPoolLoads; ++u) {
        const int tok = tb + u * TPW + sub;
        int64_t src = -1;
        if (tok < cnt) src = perm ? (int64_t)srow[tok] : t0 + tok;
        if (src >= 0) okm |= 1u << u;
        raw[u] = src >= 0 ? __ldg(xbh + src * CH) : make_uint4(0, 0, 0, 0);
      }
      if (ybh) {
#pragma unroll
        for (int u = 0; u < kPoolLoads; ++u)
          if ((okm >> u) & 1u) __stcs(ybh + (tb + u * TPW + sub) * CH, raw[u]);
      }
      // One token at a time from registers (the loads are all in flight):
      // its norm over the token's lanes, then the sums.
#pragma unroll
      for (int u = 0; u < kPoolLoads; ++u) {
        uint64_t v[NP];
        pairs16(raw[u], T(), v);
        uint64_t s2 = f2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < NP; ++e) s2 = f2_fma(v[e], v[e], s2);
        float s0, s1;
        f2_split(s2, s0, s1);
        float ss = s0 + s1;
#pragma unroll
        for (int off = CH >> 1; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
        const uint64_t inv2 = f2(inv, inv);
#pragma unroll
        for (int e = 0; e < NP; ++e) {
          ax[e] = f2_add(ax[e], v[e]);
          au[e] = f2_fma(v[e], inv2, au[e]);
        }
        if constexpr (QF != 0) {
#pragma unroll
          for (int e = 0; e < NP; ++e) {
            float lo, hi;
            f2_split(v[e], lo, hi);
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
          }
        }
      }
    }
    // Lanes c, c + CH, ... hold the same features for different tokens.
    float axs[EPL], aus[EPL];
#pragma unroll
    for (int e = 0; e < NP; ++e) {
      f2_split(ax[e], axs[2 * e], axs[2 * e + 1]);
      f2_split(au[e], aus[2 * e], aus[2 * e + 1]);
    }
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        axs[e] += __shfl_xor_sync(0xffffffffu, axs[e], off);
        aus[e] += __shfl_xor_sync(0xffffffffu, aus[e], off);
      }
    }
    float part = 0.f;
    if (lane < CH) {
      const float invc = 1.0f / (float)cnt;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int i = c * EPL + e;
        const float mv = axs[e] * invc;
        if (mean_tstride > 0) mean_out[(bh * d + i) * mean_tstride + blk] = mv;
        else mean_out[(bh * nB + blk) * (int64_t)d + i] = mv;
        part = fmaf(aus[e], aus[e], part);
      }
    }
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == 0) s_out[bh * nB + blk] = part / ((float)cnt * (float)cnt);
    if constexpr (QF != 0) {
      static_assert(sizeof(T) == 2, "8-bit codes are written from bf16 input");
      constexpr int FMT = QF - 1;
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float qmax = FMT == SA_Q_E4M3 ? 448.0f : 127.0f;
      const float qinv = amax > 0.f ? __fdiv_rn(qmax, amax) : 0.f;
      if (lane == 0) qscale[bh * nB + blk] = amax > 0.f ? __fdiv_rn(amax, qmax) : 0.f;
      uint2* y8bh = y8 + (bh * N + t0) * (int64_t)CH + c;
      for (int tok = sub; tok < cnt; tok += TPW) {
        const int64_t src = perm ? (int64_t)srow[tok] : t0 + tok;
        if (src >= 0) y8bh[tok * CH] = quant8<FMT>(__ldg(xbh + src * CH), qinv);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Row rules: the parameters of the structure-forced rows/columns, the local
// window and causal validity (the score kernel turns them into key-block
// ranges once per row).
// ---------------------------------------------------------------------------
struct RowRules {
  int64_t N, sink, txt, window, anchor;
  int bq, bk, causal;
  __device__ bool struct_row(int64_t qb) const {
    const int64_t i0 = qb * bq, i1 = min(N, (qb + 1) * bq);
    return i0 < sink || (txt > 0 && i1 - 1 >= N - txt);
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
// for every row r of the group, reading k_hat (stored transposed, feature-
// major, L2-resident, each element read once per group: a warp's load of a
// feature is one 128-byte line) and the q_hat rows from shared memory (the
// same address in every lane: broadcast, four features per load), with the
// FMAs on the packed fp32x2 pipe.  Then warp r alone finishes row r: softmax
// and TopCdf (an arg-max loop over register-resident keys when the row is
// short and few blocks are picked, else a search for the last kept
// probability: bisection over bit patterns while many candidates remain, then
// steps that test the remaining candidates' own values), the union with the
// forced parts and the causal AND -- with warp-level synchronisation only.
// Dynamic shared memory: q_hat [8][d] | scores [G][nkb rounded to 4] (fp32;
// the bisection turns a row's scores into its probabilities in place, the
// padding holding zeros) | flags [G][nkb rounded to 16] (u8).
// ---------------------------------------------------------------------------
constexpr int kMaxRowsPerCta = 8;
constexpr int kSelectRegs = 4;    // TopCdf: candidates a lane holds once at most 128 remain
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
  return (size_t)kMaxRowsPerCta * d * 4 + (size_t)G * nkb4 * 4 + (size_t)G * nkb16 +
         (size_t)kMaxRowsPerCta * kSelectRegs * 32 * 4 + (size_t)nkb16;
}

__device__ __forceinline__ float warp_max(float v) {
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

template <bool LONG>
__global__ void __launch_bounds__(kRowThreads, 2) score_topcdf_kernel(
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
  float* cand = reinterpret_cast<float*>(flags + (size_t)G * nkb16);   // [8][kSelectRegs * 32]
  uint8_t* colg = reinterpret_cast<uint8_t*>(cand + kMaxRowsPerCta * kSelectRegs * 32);   // [nkb16]
  __shared__ int s_forced[kMaxRowsPerCta];
  __shared__ int s_klim[kMaxRowsPerCta];   // last key block row r scores (-1: none)

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
    // causal validity of kb for row qb is kb * bk <= last query row of qb
    s_klim[r] = s_forced[r] ? -1
                            : (rules.causal ? (int)((min64(rules.N, (qb0 + r + 1) * rules.bq) - 1) / rules.bk)
                                            : (int)nkb - 1);
  }
  for (int i = threadIdx.x; i < rows * d; i += blockDim.x) qs[i] = qhat[(bh * nqb + qb0) * (int64_t)d + i];
  // key blocks under the similarity guard (forced columns, out of the softmax)
  for (int kb = threadIdx.x; kb < nkb; kb += blockDim.x) colg[kb] = (guard && sk[g * nkb + kb] < theta) ? 1 : 0;
  __syncthreads();
  int any_scored = 0;
  for (int r = 0; r < rows; ++r) any_scored |= !s_forced[r];

  if (any_scored) {
    // k_hat is stored transposed, [d][nkb4] per KV head: thread i takes key
    // blocks kb = i, i + 256, ..., so a warp's loads of one feature are one
    // 128-byte line.
    const float* kT = khat + g * (int64_t)d * nkb4;
    const float4* qs4 = reinterpret_cast<const float4*>(qs);
    const int nf4 = d / 4;
    // Two key blocks a thread per pass (kb and kb + 256): each shared read of
    // q_hat feeds both, and their loads are in flight together.
    auto need_of = [&](int kb) -> uint32_t {   // bit r: row r of the group scores key block kb
      uint32_t need = 0;
      if (kb < nkb && !colg[kb]) {
#pragma unroll
        for (int r = 0; r < kMaxRowsPerCta; ++r)
          if (kb <= s_klim[r]) need |= 1u << r;
      }
      return need;
    };
    if (LONG) {   // rows of at least 8 * kRowThreads blocks (the launch checks)
      // Long rows: four consecutive key blocks a thread, so a warp's 16-byte
      // load of one feature covers 128 blocks; kb pairs share a packed FMA
      // with the feature broadcast.
      const int nq = nkb4 / 4;
      const float4* kT4 = reinterpret_cast<const float4*>(kT);
      for (int q = threadIdx.x; q < nq; q += kRowThreads) {
        const uint32_t n0 = need_of(4 * q), n1 = need_of(4 * q + 1);
        const uint32_t n2 = need_of(4 * q + 2), n3 = need_of(4 * q + 3);
        uint64_t a01[kMaxRowsPerCta], a23[kMaxRowsPerCta];   // row r: blocks (4q, 4q+1), (4q+2, 4q+3)
#pragma unroll
        for (int r = 0; r < kMaxRowsPerCta; ++r) a01[r] = a23[r] = f2(0.f, 0.f);
        if (n0 | n1 | n2 | n3) {
#pragma unroll 2
          for (int e4 = 0; e4 < nf4; ++e4) {
            float4 kf[4];   // features 4 e4 .. 4 e4 + 3 of the four blocks
#pragma unroll
            for (int f = 0; f < 4; ++f) kf[f] = __ldg(kT4 + (int64_t)(4 * e4 + f) * nq + q);
#pragma unroll
            for (int r = 0; r < kMaxRowsPerCta; ++r) {
              const float4 x = qs4[r * nf4 + e4];
              const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                const uint64_t xx = f2(xv[f], xv[f]);
                a01[r] = f2_fma(xx, f2(kf[f].x, kf[f].y), a01[r]);
                a23[r] = f2_fma(xx, f2(kf[f].z, kf[f].w), a23[r]);
              }
            }
          }
        }
#pragma unroll
        for (int r = 0; r < kMaxRowsPerCta; ++r) {
          if (r < rows) {
            float s0, s1, s2, s3;
            f2_split(a01[r], s0, s1);
            f2_split(a23[r], s2, s3);
            float4 o;
            o.x = ((n0 >> r) & 1u) ? s0 * scale : -INFINITY;
            o.y = ((n1 >> r) & 1u) ? s1 * scale : -INFINITY;
            o.z = ((n2 >> r) & 1u) ? s2 * scale : -INFINITY;
            o.w = ((n3 >> r) & 1u) ? s3 * scale : -INFINITY;
            reinterpret_cast<float4*>(sc + r * nkb4)[q] = o;
          }
        }
      }
    } else {
      for (int kb0 = threadIdx.x; kb0 < nkb4; kb0 += 2 * kRowThreads) {   // the padding gets -inf
        const int kb1 = kb0 + kRowThreads;
        const uint32_t need0 = need_of(kb0), need1 = kb1 < nkb4 ? need_of(kb1) : 0u;
        // Row r's dot products as two packed partial sums each: features
        // (4e, 4e+1) and (4e+2, 4e+3) of each group of four.
        uint64_t a0[kMaxRowsPerCta], a1[kMaxRowsPerCta];
#pragma unroll
        for (int r = 0; r < kMaxRowsPerCta; ++r) a0[r] = a1[r] = f2(0.f, 0.f);
        if (need0 | need1) {
          // a block no row needs reads block kb0 instead (in bounds, discarded)
          const float* kc0 = kT + kb0;
          const float* kc1 = kT + (need1 ? kb1 : kb0);
#pragma unroll 4
          for (int e4 = 0; e4 < nf4; ++e4) {
            const int64_t o = (int64_t)(4 * e4) * nkb4;
            const uint64_t p01 = f2(__ldg(kc0 + o), __ldg(kc0 + o + nkb4));
            const uint64_t p23 = f2(__ldg(kc0 + o + 2 * nkb4), __ldg(kc0 + o + 3 * nkb4));
            const uint64_t q01 = f2(__ldg(kc1 + o), __ldg(kc1 + o + nkb4));
            const uint64_t q23 = f2(__ldg(kc1 + o + 2 * nkb4), __ldg(kc1 + o + 3 * nkb4));
#pragma unroll
            for (int r = 0; r < kMaxRowsPerCta; ++r) {
              const float4 x = qs4[r * nf4 + e4];
              const uint64_t x01 = f2(x.x, x.y), x23 = f2(x.z, x.w);
              a0[r] = f2_fma(x01, p01, a0[r]);
              a0[r] = f2_fma(x23, p23, a0[r]);
              a1[r] = f2_fma(x01, q01, a1[r]);
              a1[r] = f2_fma(x23, q23, a1[r]);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < kMaxRowsPerCta; ++r) {
          if (r < rows) {
            float lo, hi;
            f2_split(a0[r], lo, hi);
            sc[r * nkb4 + kb0] = ((need0 >> r) & 1u) ? (lo + hi) * scale : -INFINITY;
            if (kb1 < nkb4) {
              f2_split(a1[r], lo, hi);
              sc[r * nkb4 + kb1] = ((need1 >> r) & 1u) ? (lo + hi) * scale : -INFINITY;
            }
          }
        }
      }
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
  for (int i = lane; i < nkb16 / 16; i += 32) reinterpret_cast<uint4*>(fl)[i] = make_uint4(0, 0, 0, 0);
  // Float4 groups that can hold a finite score: key blocks past the row's
  // last valid one (causal) and the padding are -inf.
  const int nq_row = row_forced ? 0 : min(nkb4 / 4, (s_klim[r] + 4) / 4);
  if (!row_forced) {
    const float* srow = sc + r * nkb4;
    const float4* srow4 = reinterpret_cast<const float4*>(srow);
    float mx = -INFINITY;
    for (int q = lane; q < nq_row; q += 32) {
      const float4 v = srow4[q];
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
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
          const float pv = (sv == -INFINITY) ? 0.f : __expf(sv - mx);
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
      float4* pw4 = reinterpret_cast<float4*>(pr);
      for (int q = lane; q < nq_row; q += 32) {
        const float4 v = srow4[q];
        float4 o;
        o.x = v.x == -INFINITY ? 0.f : __expf(v.x - mx);
        o.y = v.y == -INFINITY ? 0.f : __expf(v.y - mx);
        o.z = v.z == -INFINITY ? 0.f : __expf(v.z - mx);
        o.w = v.w == -INFINITY ? 0.f : __expf(v.w - mx);
        pw4[q] = o;
      }
      __syncwarp();
      const float4* pr4 = reinterpret_cast<const float4*>(pr);
      // f(t) and the number of p whose bits exceed t, over the whole row.
      auto pass_full = [&](uint32_t t, int& count) -> float {
        float m0 = 0.f, m1 = 0.f;
        int c = 0;
        for (int q = lane; q < nq_row; q += 32) {
          const float4 v = pr4[q];
          const bool g0 = __float_as_uint(v.x) > t, g1 = __float_as_uint(v.y) > t;
          const bool g2 = __float_as_uint(v.z) > t, g3 = __float_as_uint(v.w) > t;
          m0 += (g0 ? v.x : 0.f) + (g1 ? v.y : 0.f);
          m1 += (g2 ? v.z : 0.f) + (g3 ? v.w : 0.f);
          c += (int)g0 + (int)g1 + (int)g2 + (int)g3;
        }
        float m = m0 + m1;
        for (int off = 16; off > 0; off >>= 1) m += __shfl_xor_sync(0xffffffffu, m, off);
        count = __reduce_add_sync(0xffffffffu, c);
        return m;
      };
      // The bisection starts at e = (1 - tau) / (4 n) instead of 0 (n = 4
      // nq_row entries): the p <= e sum to at most (1 - tau) / 4, and total
      // >= max p = 1, so f(e) >= tau * total + 0.75 (1 - tau) total -- above
      // the limit by far more than the rounding of the sums while 1 - tau >=
      // 1e-3 (otherwise the start stays 0).  The first pass takes the total,
      // f(0), and the number of p above e together.
      const uint32_t lo0 = (tau <= 0.999f) ? __float_as_uint(0.25f * (1.f - tau) / (float)(4 * nq_row)) : 0u;
      int c_lo = 0, c_hi = 0, c_mid = 0;   // how many p have bits above lo, hi
      float total;
      {
        float m0 = 0.f, m1 = 0.f;
        int c = 0;
        for (int q = lane; q < nq_row; q += 32) {
          const float4 v = pr4[q];
          const bool g0 = __float_as_uint(v.x) > 0u, g1 = __float_as_uint(v.y) > 0u;
          const bool g2 = __float_as_uint(v.z) > 0u, g3 = __float_as_uint(v.w) > 0u;
          m0 += (g0 ? v.x : 0.f) + (g1 ? v.y : 0.f);
          m1 += (g2 ? v.z : 0.f) + (g3 ? v.w : 0.f);
          c += (int)(__float_as_uint(v.x) > lo0) + (int)(__float_as_uint(v.y) > lo0) +
               (int)(__float_as_uint(v.z) > lo0) + (int)(__float_as_uint(v.w) > lo0);
        }
        total = m0 + m1;
        for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
        c_lo = __reduce_add_sync(0xffffffffu, c);
      }
      const float limit = tau * total;
      uint32_t lo = lo0, hi = 0x3F800000u;   // f(lo) >= limit (tau <= 1), f(hi) = 0 < limit
      float f_hi = 0.f;                     // f(hi)
      while (hi - lo > 1u && c_lo - c_hi > kSelectRegs * 32) {
        const uint32_t mid = lo + (hi - lo) / 2u;
        const float m = pass_full(mid, c_mid);
        if (m < limit) {
          hi = mid;
          f_hi = m;
          c_hi = c_mid;
        } else {
          lo = mid;
          c_lo = c_mid;
        }
      }
      if (hi - lo > 1u) {
        // At most kSelectRegs * 32 p lie in (lo, hi]: gather them (in block
        // order) into the warp's buffer, then into registers, and finish the
        // search there: f(t) = f(hi on entry) + the mass of the gathered p
        // above t.
        float* cbuf = cand + warp * kSelectRegs * 32;
        int n = 0;
        for (int kb0 = 0; kb0 < 4 * nq_row; kb0 += 32) {
          const int kb = kb0 + lane;
          const float v = kb < 4 * nq_row ? pr[kb] : 0.f;
          const uint32_t bits = __float_as_uint(v);
          const bool in = bits > lo && bits <= hi;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (in) cbuf[n + __popc(bal & ((1u << lane) - 1u))] = v;
          n += __popc(bal);
        }
        __syncwarp();
        float cv[kSelectRegs];
#pragma unroll
        for (int j = 0; j < kSelectRegs; ++j) cv[j] = lane + 32 * j < n ? cbuf[lane + 32 * j] : 0.f;
        const float f_base = f_hi;   // f(hi) on entry: every gathered p is <= hi
        // f only changes at the gathered values, so the boundary is one of
        // them (or hi): each step tests a candidate strictly inside (lo, hi),
        // taken from a rotating lane, which then leaves the interval; the
        // search ends when none is left (at most kSelectRegs * 32 steps) and
        // reaches the same hi as a bisection over the bit patterns.
        for (int step = 0;; ++step) {
          float piv = 0.f;
          bool has = false;
#pragma unroll
          for (int j = kSelectRegs - 1; j >= 0; --j) {
            const uint32_t bj = __float_as_uint(cv[j]);
            if (bj > lo && bj < hi) {
              piv = cv[j];
              has = true;
            }
          }
          const unsigned bal = __ballot_sync(0xffffffffu, has);
          if (bal == 0u) break;
          const int rot = (step * 13) & 31;
          const unsigned rb = (bal >> rot) | (bal << ((32 - rot) & 31));
          const int src = (__ffs((int)rb) - 1 + rot) & 31;
          const uint32_t mid = __float_as_uint(__shfl_sync(0xffffffffu, piv, src));
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < kSelectRegs; ++j) s += __float_as_uint(cv[j]) > mid ? cv[j] : 0.f;
          for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
          const float m = f_base + s;
          if (m < limit) {
            hi = mid;
            f_hi = m;
          } else {
            lo = mid;
          }
        }
      }
      const float above = f_hi;
      const float vstar = __uint_as_float(hi);
      uint32_t run = 0;
      const int nrow = 4 * nq_row;   // p beyond this is 0: never kept (hi > 0)
      for (int kb0 = 0; kb0 < nrow; kb0 += 32) {
        const int kb = kb0 + lane;
        const uint32_t bits = kb < nrow ? __float_as_uint(pr[kb]) : 0u;
        const bool tie = kb < nrow && bits == hi;
        const unsigned bal = __ballot_sync(0xffffffffu, tie);
        bool keep = kb < nrow && bits > hi;
        if (tie) keep = above + (float)(run + __popc(bal & ((1u << lane) - 1u))) * vstar < limit;
        if (keep) fl[kb] = 1;
        run += __popc(bal);
      }
    }
  }
  __syncwarp();
  // The row's key-block ranges, once: causally valid blocks kb <= klim; the
  // local window [w0, w1]; the structural columns (sink, anchors) kb < c0 and
  // (text) kb >= c1.
  const int64_t i0 = qb * rules.bq, i1 = min64(rules.N, (qb + 1) * rules.bq);
  const int klim = rules.causal ? (int)((i1 - 1) / rules.bk) : (int)nkb - 1;
  int w0 = 1, w1 = 0;
  if (rules.window > 0) {
    // j1 - 1 >= i0 - window + 1 and j0 <= i1 - 1, with j0 = kb * bk, j1 = min(N, j0 + bk)
    w0 = (int)max64(0, (i0 - rules.window + 1) / rules.bk);
    while (w0 > 0 && min64(rules.N, (int64_t)(w0 - 1) * rules.bk + rules.bk) - 1 >= i0 - rules.window + 1) --w0;
    while (w0 < nkb && min64(rules.N, (int64_t)w0 * rules.bk + rules.bk) - 1 < i0 - rules.window + 1) ++w0;
    w1 = (int)min64(nkb - 1, (i1 - 1) / rules.bk);
  }
  const int64_t front = max64(rules.sink, rules.anchor);
  const int c0 = (int)min64(nkb, (front + rules.bk - 1) / rules.bk);   // kb * bk < front
  int c1 = (int)nkb;                                                 // last row of kb >= N - txt
  if (rules.txt > 0) {
    c1 = (int)max64(0, (rules.N - rules.txt) / rules.bk);
    while (c1 > 0 && min64(rules.N, (int64_t)c1 * rules.bk) - 1 >= rules.N - rules.txt) --c1;
    while (c1 < nkb && min64(rules.N, (int64_t)(c1 + 1) * rules.bk) - 1 < rules.N - rules.txt) ++c1;
  }
  int cnt = 0, first = 0x7fffffff;
  uint8_t* mrow = mask + u * nkb;
  auto keep_of = [&](int kb, bool picked) -> bool {
    const bool col = kb < c0 || kb >= c1 || colg[kb];
    const bool keep = kb <= klim && (row_forced || picked || col || (kb >= w0 && kb <= w1));
    if (keep) {
      ++cnt;
      first = min(first, kb);
    }
    return keep;
  };
  if ((nkb & 3) == 0 && (reinterpret_cast<uintptr_t>(mask) & 3) == 0) {
    // four blocks a lane: one 32-bit read of the picks, one 32-bit store
    for (int q = lane; q < nkb / 4; q += 32) {
      const uint32_t f4 = reinterpret_cast<const uint32_t*>(fl)[q];
      uint32_t out = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) out |= (keep_of(4 * q + j, ((f4 >> (8 * j)) & 0xFFu) != 0u) ? 1u : 0u) << (8 * j);
      reinterpret_cast<uint32_t*>(mrow)[q] = out;
    }
  } else {
    for (int kb = lane; kb < nkb; kb += 32) mrow[kb] = keep_of(kb, fl[kb] != 0) ? 1 : 0;
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
// CSR: one CTA scans the row counts into row_ptr and checks capacity.  The
// counts are read kScanBatch chunks of 1024 at a time (coalesced, all loads
// of a batch in flight together); each chunk is one block-wide scan (warp
// shuffles, then one warp over the 32 warp totals) on top of the running
// total of the chunks before it.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;
constexpr int kScanBatch = 8;

__global__ void __launch_bounds__(kScanThreads) rows_scan_kernel(const int32_t* __restrict__ counts,
                                                                 int64_t R, int64_t capacity,
                                                                 int32_t* __restrict__ row_ptr,
                                                                 int64_t* kept_total, int32_t* status) {
  __shared__ int32_t wsum[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t carry = 0;   // kept blocks of all rows before the current chunk
  for (int64_t base = 0; base < R; base += (int64_t)kScanBatch * kScanThreads) {
    int32_t v[kScanBatch];
#pragma unroll
    for (int j = 0; j < kScanBatch; ++j) {
      const int64_t i = base + (int64_t)j * kScanThreads + tid;
      v[j] = i < R ? counts[i] : 0;
    }
#pragma unroll
    for (int j = 0; j < kScanBatch; ++j) {
      int32_t x = v[j];   // a chunk sums at most 1024 * 4095 blocks: int32 holds it
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += o;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      if (warp == 0) {
        int32_t y = wsum[lane];
        for (int off = 1; off < 32; off <<= 1) {
          const int32_t o = __shfl_up_sync(0xffffffffu, y, off);
          if (lane >= off) y += o;
        }
        wsum[lane] = y;
      }
      __syncthreads();
      const int64_t i = base + (int64_t)j * kScanThreads + tid;
      const int64_t excl = carry + (warp > 0 ? wsum[warp - 1] : 0) + (x - v[j]);
      if (i < R) row_ptr[i] = (int32_t)min64(excl, INT32_MAX);
      carry += wsum[kScanThreads / 32 - 1];
      __syncthreads();
    }
  }
  if (tid == 0) {
    row_ptr[R] = (int32_t)min64(carry, INT32_MAX);
    *kept_total = carry;
    if (carry > capacity || carry > INT32_MAX) raise_status(status, SA_ERR_CAPACITY);
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

// The same for rows of a multiple of 16 blocks: a lane reads 16 flag bytes
// at once (a warp covers 512 key blocks per load), and the lanes' kept
// counts are placed by a warp exclusive scan.
__global__ void fill_cols_vec_kernel(const uint8_t* __restrict__ mask, int64_t R, int64_t nkb,
                                     const int32_t* __restrict__ row_ptr, int64_t capacity,
                                     int32_t* __restrict__ col_idx) {
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= R) return;
  const int64_t lo = row_ptr[warp];
  const int64_t hi = row_ptr[warp + 1];
  if (hi > capacity) return;  // capacity error already raised
  const uint4* mrow = reinterpret_cast<const uint4*>(mask + warp * nkb);
  const int64_t nv = nkb / 16;
  int64_t pos = lo;
  for (int64_t v0 = 0; v0 < nv; v0 += 32) {
    const int64_t vi = v0 + lane;
    const uint4 m = vi < nv ? __ldg(mrow + vi) : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {m.x, m.y, m.z, m.w};
    uint32_t bits = 0;   // bit j: flag byte j of the 16 is set
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int j = 0; j < 4; ++j) bits |= (((w[q] >> (8 * j)) & 0xFFu) != 0u ? 1u : 0u) << (4 * q + j);
    const int c = __popc(bits);
    int x = c;
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += o;
    }
    int64_t p = pos + (x - c);
    while (bits) {
      const int j = __ffs(bits) - 1;
      col_idx[p++] = (int32_t)(vi * 16 + j);
      bits &= bits - 1u;
    }
    pos += __shfl_sync(0xffffffffu, x, 31);
  }
}

// Work order: stable LSD radix sort of rows by key = 4095 - count, i.e.
// descending count, ties by ascending row index.  One CTA.
//
// order_smem_kernel (R <= kOrderSmemRows): two passes of 6 bits, with the
// keys and the intermediate sequence as 16-bit values in shared memory; only
// the second pass writes `order`.  Warp w owns a contiguous range of the
// current sequence and walks it 32 rows at a time: the lanes holding the same
// digit find one another with a match, their leader adds the group's size to
// the warp's count of that digit, and in the scatter each lane's slot is the
// warp's running offset of its digit plus its rank among the lower lanes of
// its group.  The offsets of entry (digit, warp) are every entry of smaller
// digits plus the same digit's entries of smaller warps, so every pass is
// stable.  With order_group = g > 0 one CTA sorts each group of g * nqb rows
// (at most kOrderSmemRows).  order_kernel (one global order of more rows):
// per-thread histograms and three passes of 4 bits through `tmp` and `order`
// in global memory.
constexpr int kOrderSmemRows = 32768;
constexpr int kOrderSmemThreads = 1024;
constexpr int kOrderSmemWarps = kOrderSmemThreads / 32;
constexpr int kWhistStride = 65;   // a warp's 64 digit counts, padded

size_t order_smem_bytes(int64_t R) {
  return (size_t)kOrderSmemWarps * kWhistStride * 4 + (size_t)R * 2 * 2;
}

__global__ void __launch_bounds__(kOrderSmemThreads) order_smem_kernel(const int32_t* __restrict__ counts,
                                                                       int64_t R, int64_t seg_rows,
                                                                       int32_t* __restrict__ order) {
  extern __shared__ uint32_t dyn[];
  uint32_t* whist = dyn;                                                       // [warps][65]
  uint16_t* skey = reinterpret_cast<uint16_t*>(dyn + kOrderSmemWarps * kWhistStride);   // [seg_rows]
  uint16_t* seq = skey + seg_rows;                                             // [seg_rows] after pass 0
  __shared__ uint32_t wsum[kOrderSmemWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this CTA's segment: rows [base, base + n)
  const int64_t base = (int64_t)blockIdx.x * seg_rows;
  const int n = (int)min64(seg_rows, R - base);
  counts += base;
  order += base;
  const int per = (n + kOrderSmemWarps - 1) / kOrderSmemWarps;
  const int beg = min(n, warp * per), end = min(n, beg + per);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t* wh = whist + warp * kWhistStride;
  for (int i = tid; i < n; i += kOrderSmemThreads) skey[i] = (uint16_t)(4095u - (uint32_t)counts[i]);
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = 6 * pass;
    wh[lane] = 0;
    wh[lane + 32] = 0;
    __syncthreads();   // keys (pass 0) or the sequence (pass 1) are complete
    for (int i0 = beg; i0 < end; i0 += 32) {
      const int i = i0 + lane;
      const bool valid = i < end;
      const int row = valid ? (pass == 0 ? i : (int)seq[i]) : 0;
      const uint32_t dgt = valid ? ((uint32_t)skey[row] >> shift) & 63u : 64u;
      const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
      if (valid && (peers & lt) == 0u) wh[dgt] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    // Exclusive scan in (digit, warp) order: thread t holds entries 2t, 2t + 1.
    {
      const int e0 = 2 * tid, e1 = e0 + 1;
      uint32_t* c0 = whist + (e0 & 31) * kWhistStride + (e0 >> 5);
      uint32_t* c1 = whist + (e1 & 31) * kWhistStride + (e1 >> 5);
      const uint32_t a = *c0, b = *c1;
      uint32_t x = a + b;
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += o;
      }
      if (lane == 31) wsum[warp] = x;
      __syncthreads();
      if (warp == 0) {
        uint32_t y = wsum[lane];
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t o = __shfl_up_sync(0xffffffffu, y, off);
          if (lane >= off) y += o;
        }
        wsum[lane] = y;
      }
      __syncthreads();
      const uint32_t ex = (warp > 0 ? wsum[warp - 1] : 0u) + x - (a + b);
      *c0 = ex;
      *c1 = ex + a;
    }
    __syncthreads();
    for (int i0 = beg; i0 < end; i0 += 32) {
      const int i = i0 + lane;
      const bool valid = i < end;
      const int row = valid ? (pass == 0 ? i : (int)seq[i]) : 0;
      const uint32_t dgt = valid ? ((uint32_t)skey[row] >> shift) & 63u : 64u;
      const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
      if (valid) {
        const uint32_t slot = wh[dgt] + __popc(peers & lt);
        if (pass == 0) seq[slot] = (uint16_t)row;
        else order[slot] = (int32_t)(base + row);
      }
      __syncwarp();
      if (valid && (peers & lt) == 0u) wh[dgt] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
  }
}

constexpr int kOrderThreads = 1024;
constexpr int kOrderWarps = kOrderThreads / 32;
constexpr int kHistStride = 17;   // a thread's 16 digit counts, padded

__global__ void __launch_bounds__(kOrderThreads) order_kernel(const int32_t* __restrict__ counts,
                                                              int64_t R, int32_t* __restrict__ tmp,
                                                              int32_t* __restrict__ order) {
  extern __shared__ uint32_t hist[];                      // [thread][17]: 16 digits, padded
  __shared__ uint32_t wtot[kOrderWarps][16];              // per-warp digit totals, then warp offsets
  __shared__ uint32_t dtot[16];                           // digit totals
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* my = hist + tid * kHistStride;
  const int64_t per = (R + kOrderThreads - 1) / kOrderThreads;
  const int64_t beg = tid * per, end = min(R, beg + per);
  auto key_of = [&](int32_t row) -> uint32_t { return 4095u - (uint32_t)counts[row]; };
  for (int pass = 0; pass < 3; ++pass) {
    // rows in natural order first; pass 0 writes order, pass 1 tmp, pass 2 order
    const int32_t* src = pass == 0 ? nullptr : (pass == 1 ? order : tmp);
    int32_t* dst = pass == 1 ? tmp : order;
    const int shift = 4 * pass;
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) my[dgt] = 0;
    for (int64_t i = beg; i < end; ++i) {
      const int32_t row = src ? src[i] : (int32_t)i;
      my[(key_of(row) >> shift) & 15u] += 1;
    }
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

sa_status launch_lists(const sa_shape& s, int bq, int bk, int order_group, int32_t* counts, int32_t* tmp,
                       sa_mask& out, cudaStream_t st) {
  const int64_t R = s.B * s.Hq * out.nqb;
  rows_scan_kernel<<<1, 1024, 0, st>>>(counts, R, out.col_capacity, out.row_ptr, out.kept_total,
                                       out.status);
  if (sa_status e = check_launch("rows_scan_kernel")) return e;
  const int64_t warps_per_block = 8;
  const unsigned fill_grid = (unsigned)ceil_div(R, warps_per_block);
  if (out.nkb % 16 == 0 && reinterpret_cast<uintptr_t>(out.block_mask) % 16 == 0)
    fill_cols_vec_kernel<<<fill_grid, 32 * warps_per_block, 0, st>>>(out.block_mask, R, out.nkb, out.row_ptr,
                                                                      out.col_capacity, out.col_idx);
  else
    fill_cols_kernel<<<fill_grid, 32 * warps_per_block, 0, st>>>(out.block_mask, R, out.nkb, out.row_ptr,
                                                                  out.col_capacity, out.col_idx);
  if (sa_status e = check_launch("fill_cols_kernel")) return e;
  // Work order: one sort over all rows, or one per group of order_group heads.
  const int64_t seg = order_group > 0 ? min64(R, (int64_t)order_group * out.nqb) : R;
  const int64_t nseg = ceil_div(R, seg);
  if (seg <= kOrderSmemRows) {
    const size_t smem = order_smem_bytes(seg);
    if (cudaFuncSetAttribute(order_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(order_smem_kernel) failed");
    order_smem_kernel<<<(unsigned)nseg, kOrderSmemThreads, smem, st>>>(counts, R, seg, out.order);
    return check_launch("order_smem_kernel");
  }
  if (nseg != 1) return set_error(SA_ERR_UNSUPPORTED, "order_group * nqb must be <= %d", kOrderSmemRows);
  const size_t hist_bytes = (size_t)kHistStride * kOrderThreads * sizeof(uint32_t);
  if (cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hist_bytes) !=
      cudaSuccess)
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

// Persistent grid: as many CTAs as fit on the device at once (at most one
// warp per unit).
template <typename K>
sa_status pool_grid(K kernel, int64_t units, unsigned* grid) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kPoolThreads, 0) != cudaSuccess ||
      per_sm < 1)
    return set_error(SA_ERR_CUDA, "pool_cossim_kernel does not fit on the device");
  *grid = (unsigned)min64(ceil_div(units, kPoolWarps), (int64_t)sms * per_sm);
  return SA_OK;
}

template <typename T, int CH, int QF>
sa_status launch_pool_ch(const PoolJob& j0, const PoolJob& j1, int64_t N, const int32_t* perm, int32_t* status,
                         cudaStream_t st) {
  unsigned grid = 0;
  if (sa_status e = pool_grid(pool_cossim_kernel<T, CH, QF>, j0.BH * j0.nB + j1.BH * j1.nB, &grid)) return e;
  pool_cossim_kernel<T, CH, QF><<<grid, kPoolThreads, 0, st>>>(j0, j1, N, perm, status);
  return check_launch("pool_cossim_kernel");
}

// Q and K pooled in one launch (plain or with their reordered copies).
template <typename T>
sa_status launch_pool(const PoolJob& jq, const PoolJob& jk, int64_t N, int d, const int32_t* perm, int32_t* status,
                      cudaStream_t st) {
  switch (d / (16 / (int)sizeof(T))) {   // 16-byte chunks per token (validated: a power of two <= 32)
    case 1: return launch_pool_ch<T, 1, 0>(jq, jk, N, perm, status, st);
    case 2: return launch_pool_ch<T, 2, 0>(jq, jk, N, perm, status, st);
    case 4: return launch_pool_ch<T, 4, 0>(jq, jk, N, perm, status, st);
    case 8: return launch_pool_ch<T, 8, 0>(jq, jk, N, perm, status, st);
    case 16: return launch_pool_ch<T, 16, 0>(jq, jk, N, perm, status, st);
    case 32: return launch_pool_ch<T, 32, 0>(jq, jk, N, perm, status, st);
    default: return set_error(SA_ERR_UNSUPPORTED, "pooling: d must give a power-of-two count <= 32 of 16-byte chunks");
  }
}

// Pooling with 8-bit codes and block scales instead of the reordered copies
// (bf16, d = 128: 16 chunks).
sa_status launch_pool_codes(const PoolJob& jq, const PoolJob& jk, int64_t N, int d, const int32_t* perm,
                            int32_t fmt, int32_t* status, cudaStream_t st) {
  if (d != 128) return set_error(SA_ERR_UNSUPPORTED, "8-bit codes need d = 128");
  if (fmt == SA_Q_E4M3) return launch_pool_ch<uint16_t, 16, 1 + SA_Q_E4M3>(jq, jk, N, perm, status, st);
  return launch_pool_ch<uint16_t, 16, 1 + SA_Q_INT8>(jq, jk, N, perm, status, st);
}

}  // namespace

size_t predict_ws_bytes(const sa_shape& s, int bq, int bk, size_t off[6]) {
  const int64_t nqb = ceil_div(s.N, bq), nkb = ceil_div(s.N, bk);
  const int64_t R = s.B * s.Hq * nqb;
  size_t o = 0;
  const int64_t nkb4 = (nkb + 3) / 4 * 4;
  const size_t sizes[6] = {(size_t)(s.B * s.Hq * nqb * s.d) * 4, (size_t)(s.B * s.Hkv * nkb4 * s.d) * 4,
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
  const int64_t nkb4 = (nkb + 3) / 4 * 4;   // row stride of the transposed k_hat
  if (cudaMemsetAsync(out.status, 0, sizeof(int32_t), st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync(status) failed");
  sa_status e;
  PoolJob jq{q, s.B * s.Hq, p.bq, (int)nqb, w.qhat, 0, w.sq, q_r, nullptr, nullptr};
  PoolJob jk{k, s.B * s.Hkv, p.bk, (int)nkb, w.khat, nkb4, w.sk, k_r, nullptr, nullptr};
  if (codes) {   // bf16 input: codes and scales instead of reordered copies
    jq.y = jk.y = nullptr;
    jq.y8 = static_cast<uint2*>(codes->q8);
    jq.qscale = codes->q_scales;
    jk.y8 = static_cast<uint2*>(codes->k8);
    jk.qscale = codes->k_scales;
    if ((e = launch_pool_codes(jq, jk, s.N, (int)s.d, perm, codes->format, out.status, st))) return e;
  } else if (s.dtype == SA_BF16) {
    if ((e = launch_pool<uint16_t>(jq, jk, s.N, (int)s.d, perm, out.status, st))) return e;
  } else {
    if ((e = launch_pool<float>(jq, jk, s.N, (int)s.d, perm, out.status, st))) return e;
  }
  int P2 = 1;
  while (P2 < nkb) P2 <<= 1;
  const int G = score_rows_per_cta(P2);
  const size_t smem = score_smem_bytes((int)s.d, nkb, P2, G);
  // Rows of at least 2048 blocks (8 x 256, counted with the padding to 4)
  // score four blocks a thread; shorter rows two.
  const bool long_rows = nkb4 >= 8 * kRowThreads;
  auto kern = long_rows ? score_topcdf_kernel<true> : score_topcdf_kernel<false>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(score_topcdf_kernel) failed");
  }
  dim3 grid((unsigned)ceil_div(nqb, G), (unsigned)(s.B * s.Hq));
  kern<<<grid, kRowThreads, smem, st>>>(w.qhat, w.khat, w.sq, w.sk, s.Hq, s.Hkv, nqb, nkb, (int)s.d, P2, G, p.tau,
                                        p.theta, make_rules(s, p), out.block_mask, w.counts, out.status);
  if ((e = check_launch("score_topcdf_kernel"))) return e;
  return launch_lists(s, p.bq, p.bk, p.order_group, w.counts, w.tmp, out, st);
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
  return launch_lists(s, bq, bk, 0, counts, tmp, out, st);
}

}  // namespace sa
