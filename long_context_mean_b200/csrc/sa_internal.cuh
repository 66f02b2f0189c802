// Internal declarations shared by the CUDA translation units of
// libsparseattn.so.  Nothing here is part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// ---------------------------------------------------------------------------
// Host-side error reporting (thread-local message, see abi.cu)
// ---------------------------------------------------------------------------
sa_status set_error(sa_status code, const char* fmt, ...);
sa_status check_launch(const char* what);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// 8-bit codes of two bf16 values (low, high half of w), low byte first:
// INT8 rint(x * inv) clamped to [-127, 127]; E4M3 by the saturating
// hardware conversion of x * inv (ties to even).  Used by the standalone
// quantisation kernel and by the pooling pass that writes codes directly.
__device__ __forceinline__ uint32_t quant_int8(uint32_t bits16, float inv) {
  const float f = __uint_as_float(bits16 << 16);
  int q = __float2int_rn(f * inv);
  q = max(-127, min(127, q));
  return (uint32_t)(uint8_t)(int8_t)q;
}
template <int FMT>
__device__ __forceinline__ uint32_t quant2(uint32_t w, float inv) {
  if constexpr (FMT == SA_Q_E4M3) {
    const float2 f = make_float2(__uint_as_float(w << 16) * inv, __uint_as_float(w & 0xFFFF0000u) * inv);
    return (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
  } else {
    return quant_int8(w & 0xFFFFu, inv) | (quant_int8(w >> 16, inv) << 8);
  }
}
// Eight bf16 values (one 16-byte vector) to eight codes.
template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, float inv) {
  return make_uint2(quant2<FMT>(v.x, inv) | (quant2<FMT>(v.y, inv) << 16),
                    quant2<FMT>(v.z, inv) | (quant2<FMT>(v.w, inv) << 16));
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<uint16_t> {
  static __device__ __forceinline__ float load(const uint16_t* p) { return bf16_to_f32(__ldg(p)); }
  static __device__ __forceinline__ void store(uint16_t* p, float v) { *p = f32_to_bf16_rne(v); }
};

// Unpack a 16-byte vector of elements into floats (8 bf16 or 4 fp32).
__device__ __forceinline__ void unpack16(const uint4& u, uint16_t, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack16(const uint4& u, float, float* f) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------------------
// Launch entry points implemented in the .cu files (called from abi.cu after
// argument validation).
// ---------------------------------------------------------------------------
sa_status launch_layout(const sa_layout_desc& d, int32_t* perm, int32_t* inv, void* ws,
                        cudaStream_t st);
size_t layout_ws_bytes(const sa_layout_desc& d);

// pstride: 0 = one perm for every outer index; N = perm[o * N + n], one per outer index.
sa_status launch_reorder(const int32_t* perm, const void* src, void* dst, int64_t outer,
                         int64_t N, int64_t row_bytes, bool scatter, cudaStream_t st, int64_t pstride = 0);

struct PredictWs {
  float* qhat;     // [B*Hq, nqb, d]
  float* khat;     // [B*Hkv, d, nkb4] (transposed; nkb4 = nkb rounded up to 4)
  float* sq;       // [B*Hq, nqb]
  float* sk;       // [B*Hkv, nkb]
  int32_t* counts; // [B*Hq*nqb]
  int32_t* tmp;    // [B*Hq*nqb] radix-sort scratch
};
size_t predict_ws_bytes(const sa_shape& s, int bq, int bk, size_t offsets[6]);
PredictWs predict_ws_carve(void* ws, const sa_shape& s, int bq, int bk);
size_t lists_ws_bytes(const sa_shape& s, int bq, int bk);

// With perm (nullable), q and k are in the original token order: the pooling
// pass reads row perm[n] for token n and writes the reordered copies q_r, k_r.
// Optional 8-bit outputs of the pooling pass (instead of reordered bf16
// copies): the codes and block scales of Q (per query block) and K (per key
// block) in `format`.
struct PoolCodes {
  int32_t format;
  void* q8;
  float* q_scales;
  void* k8;
  float* k_scales;
};
sa_status launch_predict(const void* q, const void* k, const sa_shape& s,
                         const sa_mask_params& p, const PredictWs& w, sa_mask& out,
                         cudaStream_t st, const int32_t* perm = nullptr, void* q_r = nullptr,
                         void* k_r = nullptr, const PoolCodes* codes = nullptr);
sa_status launch_mask_from_blocks(const uint8_t* in, const sa_shape& s, int bq, int bk,
                                  int causal, int32_t* counts, int32_t* tmp, sa_mask& out,
                                  cudaStream_t st);

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  const int32_t* out_perm;  // nullptr = rows stored in place
  int64_t perm_stride;      // 0: out_perm shared by all heads; N: out_perm[bh * N + n]
  const float* tile_scale;  // non-null: q, k are 8-bit codes and this holds each kept tile's
                            // log2-domain score scale in CSR order (tensor-core kernel only)
  int32_t qfmt;             // the codes' format: SA_Q_INT8 or SA_Q_E4M3
  uint8_t* skip_log;
  const int32_t* row_ptr;   // nullptr = dense (every causally valid block)
  const int32_t* col_idx;
  int64_t col_capacity;     // entries col_idx holds: a row whose list reaches past it is not
                            // computed (the mask's builder raised SA_ERR_CAPACITY)
  const int32_t* order;     // nullptr = natural row order
  int32_t* status;
  int32_t* counter;         // attention workspace: the work counter
  int64_t B, Hq, Hkv, N, d, dv;
  int32_t dtype;
  int32_t bq, bk, causal;
  int64_t nqb, nkb;
  float scale;
  float lambda;
  int32_t flags;            // SA_FLAG_* of the call
};
sa_status launch_attn_simt(const AttnArgs& a, cudaStream_t st);
sa_status launch_head_placement(int64_t T, int64_t P, int64_t n, const int32_t* kinds, int64_t heads, int bq,
                                int bk, int32_t* perms, uint8_t* mask, int32_t* status, cudaStream_t st);
bool rows_attn_supported(int64_t d, int64_t dv, int64_t N, int bk);
sa_status launch_rows_attn(const void* q, const void* k, const void* v, const sa_shape& s, const int32_t* rows,
                           int64_t nrows, const int32_t* perms, const uint8_t* block_mask, int bq, int bk,
                           float scale, float* out, float* lse, int32_t* status, cudaStream_t st);
sa_status launch_rows_mse(const void* ref, const void* x, const int32_t* rows, int64_t nrows, int64_t BH, int64_t N,
                          int64_t dv, int32_t dtype, double* out, int32_t* status, cudaStream_t st);
sa_status launch_quant_blocks(const void* x, int64_t heads, int64_t N, int64_t d, int rows, int32_t fmt, void* x8,
                              float* scales, cudaStream_t st);
bool quant_blocks_fits(int64_t d, int rows);
sa_status launch_tile_scales(const sa_mask& m, int64_t B, int64_t Hq, int64_t Hkv, const float* qs, const float* ks,
                             float scale_log2, float* ts, cudaStream_t st);
sa_status launch_l1(const void* ref, const void* x, int64_t n, int32_t dtype, double* sums, cudaStream_t st);
sa_status launch_attn_tc(const AttnArgs& a, cudaStream_t st);
bool attn_tc_supported(const sa_shape& s, int bq, int bk);

}  // namespace sa
