// The C ABI of libsparseattn.so: argument validation, workspace sizing and
// dispatch to the kernels.  Every check here runs on the host before any
// work is enqueued; nothing allocates device memory.
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "sa_internal.cuh"

namespace sa {

namespace {
thread_local char g_err[768] = "";
}

sa_status set_error(sa_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

sa_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SA_OK;
}

}  // namespace sa

using namespace sa;

namespace {

sa_status check_shape(const sa_shape* s) {
  if (!s) return set_error(SA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->N <= 0 || s->d <= 0 || s->dv <= 0)
    return set_error(SA_ERR_INVALID_ARG, "shape sizes must be positive");
  if (s->Hq % s->Hkv != 0) return set_error(SA_ERR_INVALID_ARG, "Hq must be a multiple of Hkv");
  if (s->dtype != SA_BF16 && s->dtype != SA_FP32) return set_error(SA_ERR_INVALID_ARG, "unknown dtype");
  if (s->N > (int64_t)INT32_MAX / 2) return set_error(SA_ERR_UNSUPPORTED, "N too large");
  return SA_OK;
}

sa_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return set_error(SA_ERR_CUDA, "no usable CUDA device");
  }
  return SA_OK;
}

bool is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

int elem_size(int32_t dtype) { return dtype == SA_BF16 ? 2 : 4; }

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

sa_status check_blocks(int32_t bq, int32_t bk, int64_t N) {
  if (bq < 1 || bq > 128 || bk < 1 || bk > 128)
    return set_error(SA_ERR_INVALID_ARG, "bq and bk must lie in [1, 128]");
  if (ceil_div(N, bk) > 4095) return set_error(SA_ERR_UNSUPPORTED, "N / bk must be <= 4095");
  return SA_OK;
}

sa_status check_mask_out(const sa_mask* m) {
  if (!m) return set_error(SA_ERR_INVALID_ARG, "mask is NULL");
  if (!m->block_mask || !m->row_ptr || !m->col_idx || !m->order || !m->kept_total || !m->status)
    return set_error(SA_ERR_INVALID_ARG, "mask buffers must all be non-NULL");
  if (m->col_capacity <= 0) return set_error(SA_ERR_INVALID_ARG, "mask col_capacity must be positive");
  return SA_OK;
}

sa_status check_predict_dims(const sa_shape* s) {
  const int es = elem_size(s->dtype);
  if (!is_pow2(s->d) || s->d > 256 || (s->d * es) % 16 != 0 || (s->d * es) / 16 > 32)
    return set_error(SA_ERR_UNSUPPORTED,
                     "mask prediction needs d a power of two, d*elem_size a multiple of 16, d <= 256");
  return SA_OK;
}

}  // namespace

extern "C" {

const char* sa_version(void) { return "libsparseattn 0.1 (sm_100a)"; }

const char* sa_last_error(void) { return g_err; }

int32_t sa_attn_kernel_path(const sa_shape* shape, int32_t bq, int32_t bk, int32_t flags) {
  if (check_shape(shape) != SA_OK) return -1;
  if (bq < 1 || bq > 128 || bk < 1 || bk > 128) return -1;
  if (!(flags & SA_FLAG_FORCE_SIMT) && attn_tc_supported(*shape, bq, bk)) return 1;
  const size_t smem = ((size_t)bq * shape->dv + (size_t)bq * bk + 3 * (size_t)bq) * 4;
  return smem <= 227 * 1024 ? 0 : -1;
}

size_t sa_attn_workspace(void) { return 256; }

size_t sa_layout_workspace(const sa_layout_desc* desc) {
  if (!desc) return 0;
  return layout_ws_bytes(*desc);
}

sa_status sa_layout_build(const sa_layout_desc* desc, int32_t* perm, int32_t* inv, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!desc || !perm || !inv) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_layout_build");
  const sa_layout_desc& d = *desc;
  if (d.T < 1 || d.H < 1 || d.W < 1 || d.txt_len < 0 || d.sink_frames < 0 || d.sink_frames > d.T)
    return set_error(SA_ERR_INVALID_ARG, "bad layout sizes");
  if (d.T * d.H * d.W + d.txt_len > (int64_t)INT32_MAX / 2)
    return set_error(SA_ERR_UNSUPPORTED, "too many tokens");
  if (d.mode != SA_ORDER_IDENTITY && d.mode != SA_ORDER_WINDOW && d.mode != SA_ORDER_HILBERT)
    return set_error(SA_ERR_INVALID_ARG, "unknown layout mode");
  if (d.mode == SA_ORDER_WINDOW && (d.win[0] < 1 || d.win[1] < 1 || d.win[2] < 1))
    return set_error(SA_ERR_INVALID_ARG, "window sizes must be positive");
  if (d.mode == SA_ORDER_HILBERT) {
    const int64_t m = std::max(std::max(d.T - d.sink_frames, d.H), d.W);
    if (m > 512) return set_error(SA_ERR_UNSUPPORTED, "Hilbert layout supports dimensions up to 512");
    if (!ws || ws_bytes < layout_ws_bytes(d) || (uintptr_t)ws % 256)
      return set_error(SA_ERR_WORKSPACE, "Hilbert layout needs %zu bytes of 256-byte aligned workspace",
                       layout_ws_bytes(d));
  }
  if (sa_status e = check_device()) return e;
  return launch_layout(d, perm, inv, ws, static_cast<cudaStream_t>(stream));
}

static sa_status reorder_common(const int32_t* perm, const void* src, void* dst, int64_t outer,
                                int64_t N, int64_t row, int32_t dtype, bool scatter, void* stream) {
  if (!perm || !src || !dst) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_reorder");
  if (outer <= 0 || N <= 0 || row <= 0) return set_error(SA_ERR_INVALID_ARG, "sizes must be positive");
  if (dtype != SA_BF16 && dtype != SA_FP32) return set_error(SA_ERR_INVALID_ARG, "unknown dtype");
  if (src == dst) return set_error(SA_ERR_INVALID_ARG, "reorder cannot run in place");
  const int64_t bytes = row * elem_size(dtype);
  if ((uintptr_t)src % 2 || (uintptr_t)dst % 2) return set_error(SA_ERR_INVALID_ARG, "misaligned tensor");
  if (sa_status e = check_device()) return e;
  return launch_reorder(perm, src, dst, outer, N, bytes, scatter, static_cast<cudaStream_t>(stream));
}

sa_status sa_reorder(const int32_t* perm, const void* x, void* y, int64_t outer, int64_t N, int64_t row,
                     int32_t dtype, void* stream) {
  return reorder_common(perm, x, y, outer, N, row, dtype, false, stream);
}

sa_status sa_unreorder(const int32_t* perm, const void* y, void* x, int64_t outer, int64_t N,
                       int64_t row, int32_t dtype, void* stream) {
  return reorder_common(perm, y, x, outer, N, row, dtype, true, stream);
}

size_t sa_predict_mask_workspace(const sa_shape* shape, const sa_mask_params* p) {
  if (check_shape(shape) != SA_OK || !p || p->bq < 1 || p->bk < 1) return 0;
  size_t off[6];
  return predict_ws_bytes(*shape, p->bq, p->bk, off);
}

int32_t sa_order_group_hint(const sa_shape* shape) {
  if (check_shape(shape) != SA_OK) return -1;
  const double kv_head = (double)shape->N * (double)(shape->d + shape->dv) * elem_size(shape->dtype);
  const double lo = 32.0 * 1024 * 1024, hi = 96.0 * 1024 * 1024;
  if (kv_head < lo) return 0;
  const int64_t rep = shape->Hq / shape->Hkv;   // query heads per KV head
  const int64_t heads = shape->B * shape->Hq;
  int64_t g = 1;
  while (2 * g <= heads && (double)ceil_div(2 * g, rep) * kv_head <= hi) g *= 2;
  return (int32_t)g;
}

sa_status sa_predict_mask_ws_layout(const sa_shape* shape, const sa_mask_params* p, size_t offsets[6]) {
  if (sa_status e = check_shape(shape)) return e;
  if (!p || !offsets || p->bq < 1 || p->bk < 1) return set_error(SA_ERR_INVALID_ARG, "bad arguments");
  predict_ws_bytes(*shape, p->bq, p->bk, offsets);
  return SA_OK;
}

namespace {
// Validation shared by the two prediction entry points; fills the mask's
// geometry and the workspace carve-up.
sa_status predict_prepare(const char* who, const void* q, const void* k, const sa_shape* shape,
                          const sa_mask_params* params, void* ws, size_t ws_bytes, sa_mask* out) {
  if (sa_status e = check_shape(shape)) return e;
  if (!q || !k || !params) return set_error(SA_ERR_INVALID_ARG, "NULL argument to %s", who);
  const sa_mask_params& p = *params;
  if (sa_status e = check_blocks(p.bq, p.bk, shape->N)) return e;
  if (sa_status e = check_predict_dims(shape)) return e;
  if (!(p.tau > 0.f && p.tau <= 1.f)) return set_error(SA_ERR_INVALID_ARG, "tau must lie in (0, 1]");
  if (std::isnan(p.theta)) return set_error(SA_ERR_INVALID_ARG, "theta is NaN");
  if (p.sink_tokens < 0 || p.txt_len < 0 || p.local_window < 0 || p.anchor_tokens < 0)
    return set_error(SA_ERR_INVALID_ARG, "token counts must be non-negative");
  if (p.causal != 0 && p.causal != 1) return set_error(SA_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (p.order_group < 0) return set_error(SA_ERR_INVALID_ARG, "order_group must be >= 0");
  if (p.order_group > 0 && (int64_t)p.order_group * ceil_div(shape->N, p.bq) > 32768)
    return set_error(SA_ERR_UNSUPPORTED, "order_group * nqb must be <= 32768");
  if (sa_status e = check_mask_out(out)) return e;
  if ((uintptr_t)q % 16 || (uintptr_t)k % 16) return set_error(SA_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
  size_t off[6];
  const size_t need = predict_ws_bytes(*shape, p.bq, p.bk, off);
  if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
    return set_error(SA_ERR_WORKSPACE, "%s needs %zu bytes of 256-byte aligned workspace", who, need);
  if (sa_status e = check_device()) return e;
  out->nqb = ceil_div(shape->N, p.bq);
  out->nkb = ceil_div(shape->N, p.bk);
  out->bq = p.bq;
  out->bk = p.bk;
  out->causal = p.causal;
  return SA_OK;
}

bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + bytes && y < x + bytes;
}
// [a, a + na) and [b, b + nb) share a byte.
bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}
}  // namespace

sa_status sa_predict_mask(const void* q, const void* k, const sa_shape* shape,
                          const sa_mask_params* params, void* ws, size_t ws_bytes, sa_mask* out,
                          void* stream) {
  if (sa_status e = predict_prepare("sa_predict_mask", q, k, shape, params, ws, ws_bytes, out)) return e;
  return launch_predict(q, k, *shape, *params, predict_ws_carve(ws, *shape, params->bq, params->bk), *out,
                        static_cast<cudaStream_t>(stream));
}

sa_status sa_reorder_predict_mask(const int32_t* perm, const void* q, const void* k, void* q_r, void* k_r,
                                  const sa_shape* shape, const sa_mask_params* params, void* ws,
                                  size_t ws_bytes, sa_mask* out, void* stream) {
  if (sa_status e = check_shape(shape)) return e;
  if (!perm || !q_r || !k_r) return set_error(SA_ERR_INVALID_ARG, "NULL perm, q_r or k_r");
  if ((uintptr_t)q_r % 16 || (uintptr_t)k_r % 16)
    return set_error(SA_ERR_INVALID_ARG, "q_r and k_r must be 16-byte aligned");
  const size_t esz = shape->dtype == SA_BF16 ? 2 : 4;
  const size_t qbytes = (size_t)(shape->B * shape->Hq * shape->N * shape->d) * esz;
  const size_t kbytes = (size_t)(shape->B * shape->Hkv * shape->N * shape->d) * esz;
  if (ranges_overlap(q, qbytes, q_r, qbytes) || ranges_overlap(k, kbytes, k_r, kbytes) ||
      ranges_overlap(q_r, qbytes, k_r, kbytes) || ranges_overlap(q, qbytes, k_r, kbytes) ||
      ranges_overlap(k, kbytes, q_r, qbytes))
    return set_error(SA_ERR_INVALID_ARG, "q_r and k_r must not overlap q, k or each other");
  if (sa_status e = predict_prepare("sa_reorder_predict_mask", q, k, shape, params, ws, ws_bytes, out)) return e;
  return launch_predict(q, k, *shape, *params, predict_ws_carve(ws, *shape, params->bq, params->bk), *out,
                        static_cast<cudaStream_t>(stream), perm, q_r, k_r);
}

sa_status sa_reorder_predict_mask_q8(const int32_t* perm, const void* q, const void* k, int32_t format, void* q8,
                                     float* q_scales, void* k8, float* k_scales, const sa_shape* shape,
                                     const sa_mask_params* params, void* ws, size_t ws_bytes, sa_mask* out,
                                     void* stream) {
  if (sa_status e = check_shape(shape)) return e;
  if (!q8 || !k8 || !q_scales || !k_scales) return set_error(SA_ERR_INVALID_ARG, "NULL code or scale array");
  if (format != SA_Q_INT8 && format != SA_Q_E4M3)
    return set_error(SA_ERR_INVALID_ARG, "format must be SA_Q_INT8 or SA_Q_E4M3");
  if (shape->dtype != SA_BF16) return set_error(SA_ERR_UNSUPPORTED, "8-bit codes are written from bf16 input");
  if ((uintptr_t)q8 % 16 || (uintptr_t)k8 % 16)
    return set_error(SA_ERR_INVALID_ARG, "q8 and k8 must be 16-byte aligned");
  if ((uintptr_t)q_scales % 4 || (uintptr_t)k_scales % 4)
    return set_error(SA_ERR_INVALID_ARG, "q_scales and k_scales must be 4-byte aligned");
  const size_t qbytes = (size_t)(shape->B * shape->Hq * shape->N * shape->d);
  const size_t kbytes = (size_t)(shape->B * shape->Hkv * shape->N * shape->d);
  if (ranges_overlap(q, 2 * qbytes, q8, qbytes) || ranges_overlap(k, 2 * kbytes, k8, kbytes) ||
      ranges_overlap(q8, qbytes, k8, kbytes) || ranges_overlap(q, 2 * qbytes, k8, kbytes) ||
      ranges_overlap(k, 2 * kbytes, q8, qbytes))
    return set_error(SA_ERR_INVALID_ARG, "q8 and k8 must not overlap q, k or each other");
  if (params && params->bq >= 1 && params->bk >= 1) {
    // The scale arrays: one float per query block (Q) and per key block (K).
    const size_t qsb = (size_t)(shape->B * shape->Hq * ceil_div(shape->N, params->bq)) * sizeof(float);
    const size_t ksb = (size_t)(shape->B * shape->Hkv * ceil_div(shape->N, params->bk)) * sizeof(float);
    const void* spans[4] = {q, k, q8, k8};
    const size_t lens[4] = {2 * qbytes, 2 * kbytes, qbytes, kbytes};
    bool bad = ranges_overlap(q_scales, qsb, k_scales, ksb) ||
               (ws && ws_bytes && (ranges_overlap(q_scales, qsb, ws, ws_bytes) ||
                                   ranges_overlap(k_scales, ksb, ws, ws_bytes)));
    for (int i = 0; i < 4; ++i)
      bad = bad || ranges_overlap(q_scales, qsb, spans[i], lens[i]) || ranges_overlap(k_scales, ksb, spans[i], lens[i]);
    if (bad)
      return set_error(SA_ERR_INVALID_ARG,
                       "q_scales and k_scales must overlap neither each other, q, k, q8, k8 nor the workspace");
  }
  if (sa_status e = predict_prepare("sa_reorder_predict_mask_q8", q, k, shape, params, ws, ws_bytes, out)) return e;
  const PoolCodes codes{format, q8, q_scales, k8, k_scales};
  return launch_predict(q, k, *shape, *params, predict_ws_carve(ws, *shape, params->bq, params->bk), *out,
                        static_cast<cudaStream_t>(stream), perm, nullptr, nullptr, &codes);
}

size_t sa_mask_from_blocks_workspace(const sa_shape* shape, int32_t bq, int32_t bk) {
  if (check_shape(shape) != SA_OK || bq < 1 || bk < 1) return 0;
  return lists_ws_bytes(*shape, bq, bk);
}

sa_status sa_mask_from_blocks(const uint8_t* block_mask, const sa_shape* shape, int32_t bq, int32_t bk,
                              int32_t causal, void* ws, size_t ws_bytes, sa_mask* out, void* stream) {
  if (sa_status e = check_shape(shape)) return e;
  if (!block_mask) return set_error(SA_ERR_INVALID_ARG, "block_mask is NULL");
  if (sa_status e = check_blocks(bq, bk, shape->N)) return e;
  if (causal != 0 && causal != 1) return set_error(SA_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (sa_status e = check_mask_out(out)) return e;
  const size_t need = lists_ws_bytes(*shape, bq, bk);
  if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
    return set_error(SA_ERR_WORKSPACE, "sa_mask_from_blocks needs %zu bytes of 256-byte aligned workspace", need);
  if (sa_status e = check_device()) return e;
  out->nqb = ceil_div(shape->N, bq);
  out->nkb = ceil_div(shape->N, bk);
  out->bq = bq;
  out->bk = bk;
  out->causal = causal;
  const int64_t R = shape->B * shape->Hq * out->nqb;
  int32_t* counts = static_cast<int32_t*>(ws);
  int32_t* tmp = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align_up((size_t)R * 4, 256));
  return launch_mask_from_blocks(block_mask, *shape, bq, bk, causal, counts, tmp, *out,
                                 static_cast<cudaStream_t>(stream));
}

struct Qk8Args {
  const float* q_scales;   // [B*Hq][nqb]
  const float* k_scales;   // [B*Hkv][nkb]
  int32_t format;          // SA_Q_INT8 or SA_Q_E4M3
};

static sa_status attn_common(const void* q, const void* k, const void* v, const sa_shape* shape,
                             const sa_mask* mask, int32_t causal, float lambda, float scale, void* out,
                             float* lse, const int32_t* out_perm, uint8_t* skip_log, int32_t* status,
                             void* ws, size_t ws_bytes,
                             int32_t flags, void* stream, const Qk8Args* qk8 = nullptr) {
  if (sa_status e = check_shape(shape)) return e;
  if (!q || !k || !v || !out) return set_error(SA_ERR_INVALID_ARG, "NULL tensor argument");
  const size_t ws_need = qk8 ? sa_attn_qk8_workspace(mask) : sa_attn_workspace();
  if (!ws || ws_bytes < ws_need || (uintptr_t)ws % 256)
    return set_error(SA_ERR_WORKSPACE, "attention needs %zu bytes of 256-byte aligned workspace", ws_need);
  if (std::isnan(lambda) || lambda > 0.f)
    return set_error(SA_ERR_INVALID_ARG, "lambda must be <= 0 (or -INFINITY to disable the PV skip)");
  if (!(scale >= 0.f) || std::isinf(scale)) return set_error(SA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  AttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.out_perm = out_perm;
  if ((flags & SA_FLAG_OUT_PERM_PER_HEAD) && !out_perm)
    return set_error(SA_ERR_INVALID_ARG, "SA_FLAG_OUT_PERM_PER_HEAD needs out_perm");
  a.perm_stride = (flags & SA_FLAG_OUT_PERM_PER_HEAD) ? shape->N : 0;
  a.flags = flags;
  if (out_perm && (out == q || out == k || out == v))
    return set_error(SA_ERR_INVALID_ARG, "out must not alias an input when out_perm is given");
  a.skip_log = skip_log;
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.N = shape->N;
  a.d = shape->d;
  a.dv = shape->dv;
  a.dtype = shape->dtype;
  a.scale = scale > 0.f ? scale : 1.0f / std::sqrt((float)shape->d);
  a.lambda = lambda;
  a.counter = static_cast<int32_t*>(ws);
  if (mask) {
    if (sa_status e = check_mask_out(mask)) return e;
    if (mask->bq < 1 || mask->bq > 128 || mask->bk < 1 || mask->bk > 128 ||
        mask->nqb != ceil_div(shape->N, mask->bq) || mask->nkb != ceil_div(shape->N, mask->bk))
      return set_error(SA_ERR_INVALID_ARG, "mask does not match the shape (was it built for this shape?)");
    a.row_ptr = mask->row_ptr;
    a.col_idx = mask->col_idx;
    a.col_capacity = mask->col_capacity;
    a.order = mask->order;
    a.status = mask->status;
    a.bq = mask->bq;
    a.bk = mask->bk;
    a.causal = mask->causal;
  } else {
    a.status = status;
    a.causal = causal;
  }
  const bool tc_ok = !(flags & SA_FLAG_FORCE_SIMT) && is_sm100();
  if (qk8) {
    // 8-bit QK runs on the tensor-core kernel only: there is no other path.
    if (!qk8->q_scales || !qk8->k_scales) return set_error(SA_ERR_INVALID_ARG, "NULL scale array");
    if (qk8->format != SA_Q_INT8 && qk8->format != SA_Q_E4M3)
      return set_error(SA_ERR_INVALID_ARG, "format must be SA_Q_INT8 or SA_Q_E4M3");
    if (!(shape->dtype == SA_BF16 && shape->d == 128 && shape->dv == 128 && a.bq == 128 &&
          (a.bk == 64 || a.bk == 128)))
      return set_error(SA_ERR_UNSUPPORTED, "8-bit QK needs bf16 V, d = dv = 128, bq = 128, bk in {64, 128}");
    if (flags & SA_FLAG_FORCE_SIMT) return set_error(SA_ERR_UNSUPPORTED, "8-bit QK has no CUDA-core kernel");
    a.nqb = ceil_div(a.N, a.bq);
    a.nkb = ceil_div(a.N, a.bk);
    if (sa_status e = check_device()) return e;
    if (!tc_ok) return set_error(SA_ERR_UNSUPPORTED, "8-bit QK needs an sm_100 device");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* ts = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
    if (sa_status e = launch_tile_scales(*mask, a.B, a.Hq, a.Hkv, qk8->q_scales, qk8->k_scales,
                                         a.scale * 1.4426950408889634f, ts, st))
      return e;
    a.tile_scale = ts;
    a.qfmt = qk8->format;
    return launch_attn_tc(a, st);
  }
  if (!mask) {
    if (tc_ok && attn_tc_supported(*shape, 128, 64)) {
      a.bq = 128;
      a.bk = 64;
    } else {
      a.bq = 64;
      a.bk = 64;
    }
  }
  a.nqb = ceil_div(a.N, a.bq);
  a.nkb = ceil_div(a.N, a.bk);
  if (sa_status e = check_device()) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_ok && attn_tc_supported(*shape, a.bq, a.bk)) return launch_attn_tc(a, st);
  if (sa_attn_kernel_path(shape, a.bq, a.bk, SA_FLAG_FORCE_SIMT) < 0)
    return set_error(SA_ERR_UNSUPPORTED, "no attention kernel for this shape");
  return launch_attn_simt(a, st);
}

sa_status sa_block_sparse_attn(const void* q, const void* k, const void* v, const sa_shape* shape,
                               const sa_mask* mask, float lambda, float scale, void* out, float* lse,
                               const int32_t* out_perm, uint8_t* pv_skip_log, void* ws, size_t ws_bytes,
                               int32_t flags, void* stream) {
  if (!mask) return set_error(SA_ERR_INVALID_ARG, "mask is NULL");
  return attn_common(q, k, v, shape, mask, 0, lambda, scale, out, lse, out_perm, pv_skip_log, nullptr, ws,
                     ws_bytes, flags, stream);
}

size_t sa_attn_qk8_workspace(const sa_mask* mask) {
  if (!mask || mask->col_capacity < 0) return 0;
  return 256 + align_up((size_t)mask->col_capacity * sizeof(float), 256);
}

sa_status sa_quantize_blocks(const void* x, int64_t heads, int64_t N, int64_t d, int32_t rows, int32_t dtype,
                             int32_t format, void* x8, float* scales, void* stream) {
  if (!x || !x8 || !scales) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_quantize_blocks");
  if (heads < 0 || N < 1 || d < 1 || rows < 1) return set_error(SA_ERR_INVALID_ARG, "bad sizes for sa_quantize_blocks");
  if (dtype != SA_BF16) return set_error(SA_ERR_UNSUPPORTED, "sa_quantize_blocks takes bf16 input");
  if (format != SA_Q_INT8 && format != SA_Q_E4M3)
    return set_error(SA_ERR_INVALID_ARG, "format must be SA_Q_INT8 or SA_Q_E4M3");
  if (!quant_blocks_fits(d, rows))
    return set_error(SA_ERR_UNSUPPORTED, "sa_quantize_blocks needs d a multiple of 8 and rows * d <= 16384");
  if ((uintptr_t)x % 16 || (uintptr_t)x8 % 8 || (uintptr_t)scales % 4)
    return set_error(SA_ERR_INVALID_ARG, "misaligned tensor (x 16 bytes, x8 8 bytes)");
  if (sa_status e = check_device()) return e;
  return launch_quant_blocks(x, heads, N, d, rows, format, x8, scales, static_cast<cudaStream_t>(stream));
}

sa_status sa_block_sparse_attn_qk8(const void* q8, const float* q_scales, const void* k8, const float* k_scales,
                                   int32_t format, const void* v, const sa_shape* shape, const sa_mask* mask,
                                   float lambda, float scale, void* out, float* lse, const int32_t* out_perm,
                                   uint8_t* pv_skip_log, void* ws, size_t ws_bytes, int32_t flags, void* stream) {
  if (!mask) return set_error(SA_ERR_INVALID_ARG, "mask is NULL");
  if ((uintptr_t)q8 % 16 || (uintptr_t)k8 % 16 || (uintptr_t)v % 16 || (uintptr_t)out % 16)
    return set_error(SA_ERR_INVALID_ARG, "8-bit QK needs 16-byte aligned q8, k8, v, out");
  const Qk8Args qk8{q_scales, k_scales, format};
  return attn_common(q8, k8, v, shape, mask, 0, lambda, scale, out, lse, out_perm, pv_skip_log, nullptr, ws,
                     ws_bytes, flags, stream, &qk8);
}

sa_status sa_dense_attn(const void* q, const void* k, const void* v, const sa_shape* shape, int32_t causal,
                        float scale, void* out, float* lse, int32_t* status, void* ws, size_t ws_bytes,
                        int32_t flags, void* stream) {
  if (causal != 0 && causal != 1) return set_error(SA_ERR_INVALID_ARG, "causal must be 0 or 1");
  return attn_common(q, k, v, shape, nullptr, causal, -INFINITY, scale, out, lse, nullptr, nullptr, status,
                     ws, ws_bytes, flags, stream);
}

sa_status sa_read_status(const int32_t* status, void* stream) {
  if (!status) return set_error(SA_ERR_INVALID_ARG, "status is NULL");
  if (sa_status e = check_device()) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(cudaGetLastError()));
  int32_t h = 0;
  if (cudaMemcpy(&h, status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "reading the status word failed");
  if (h < 0 || h > SA_ERR_CAPACITY) return set_error(SA_ERR_CUDA, "corrupt status word %d", h);
  if (h != SA_OK) set_error((sa_status)h, "device status %d", h);
  return (sa_status)h;
}

sa_status sa_l1_error(const void* ref, const void* x, int64_t n, int32_t dtype, double* sums, void* stream) {
  if (!ref || !x || !sums) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_l1_error");
  if (dtype != SA_BF16 && dtype != SA_FP32) return set_error(SA_ERR_INVALID_ARG, "dtype must be SA_BF16 or SA_FP32");
  const int64_t per_vec = dtype == SA_BF16 ? 8 : 4;
  if (n < 0 || n % per_vec) return set_error(SA_ERR_INVALID_ARG, "n must be a non-negative multiple of %lld", (long long)per_vec);
  if ((uintptr_t)ref % 16 || (uintptr_t)x % 16 || (uintptr_t)sums % 8)
    return set_error(SA_ERR_INVALID_ARG, "ref and x must be 16-byte aligned, sums 8-byte aligned");
  if (sa_status e = check_device()) return e;
  return launch_l1(ref, x, n, dtype, sums, static_cast<cudaStream_t>(stream));
}

sa_status sa_head_placement(int64_t T, int64_t H, int64_t W, int64_t txt_len, const int32_t* kinds,
                            int64_t heads, int32_t bq, int32_t bk, int32_t* perms, uint8_t* block_mask,
                            int32_t* status, void* stream) {
  if (T < 1 || H < 1 || W < 1 || txt_len < 0 || heads < 0)
    return set_error(SA_ERR_INVALID_ARG, "sa_head_placement: T, H, W >= 1, txt_len and heads >= 0");
  if (heads > 0 && !kinds) return set_error(SA_ERR_INVALID_ARG, "kinds is NULL");
  if (block_mask && (bq < 1 || bk < 1 || bq > 128 || bk > 128))
    return set_error(SA_ERR_INVALID_ARG, "bq, bk must lie in 1..128");
  const int64_t n = T * H * W + txt_len;
  if (n > 2147483647) return set_error(SA_ERR_UNSUPPORTED, "sequence too long for int32 orders");
  if (sa_status e = check_device()) return e;
  return launch_head_placement(T, H * W, n, kinds, heads, bq, bk, perms, block_mask, status,
                               static_cast<cudaStream_t>(stream));
}

sa_status sa_reorder_heads(const int32_t* perms, const void* x, void* y, int64_t outer, int64_t N, int64_t row,
                           int32_t dtype, void* stream) {
  if (!perms || !x || !y) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_reorder_heads");
  if (outer <= 0 || N <= 0 || row <= 0) return set_error(SA_ERR_INVALID_ARG, "sizes must be positive");
  if (dtype != SA_BF16 && dtype != SA_FP32) return set_error(SA_ERR_INVALID_ARG, "unknown dtype");
  const int64_t bytes = row * elem_size(dtype);
  if (overlaps(x, y, (size_t)(outer * N * bytes)))
    return set_error(SA_ERR_INVALID_ARG, "x and y must not overlap");
  if ((uintptr_t)x % 2 || (uintptr_t)y % 2) return set_error(SA_ERR_INVALID_ARG, "misaligned tensor");
  if (sa_status e = check_device()) return e;
  return launch_reorder(perms, x, y, outer, N, bytes, false, static_cast<cudaStream_t>(stream), N);
}

sa_status sa_rows_attn(const void* q, const void* k, const void* v, const sa_shape* shape, const int32_t* rows,
                       int64_t nrows, const int32_t* perms, const uint8_t* block_mask, int32_t bq, int32_t bk,
                       float scale, float* out, float* lse, int32_t* status, void* stream) {
  if (sa_status e = check_shape(shape)) return e;
  if (!q || !k || !v || !out || (nrows > 0 && !rows)) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_rows_attn");
  if (nrows < 0) return set_error(SA_ERR_INVALID_ARG, "nrows must be >= 0");
  if (bq < 1 || bk < 1) return set_error(SA_ERR_INVALID_ARG, "bq, bk must be positive");
  if (!(scale >= 0.f) || std::isinf(scale)) return set_error(SA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (!rows_attn_supported(shape->d, shape->dv, shape->N, bk))
    return set_error(SA_ERR_UNSUPPORTED, "sa_rows_attn needs d = dv in {64, 128} and N / bk <= 4096");
  if ((uintptr_t)q % 16 || (uintptr_t)k % 16 || (uintptr_t)v % 16)
    return set_error(SA_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned");
  if (sa_status e = check_device()) return e;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)shape->d);
  return launch_rows_attn(q, k, v, *shape, rows, nrows, perms, block_mask, bq, bk, sc, out, lse, status,
                          static_cast<cudaStream_t>(stream));
}

sa_status sa_rows_mse(const void* ref, const void* x, const int32_t* rows, int64_t nrows, int64_t BH, int64_t N,
                      int64_t dv, int32_t dtype, double* out, int32_t* status, void* stream) {
  if (!ref || !x || !out || (nrows > 0 && !rows)) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_rows_mse");
  if (dtype != SA_BF16 && dtype != SA_FP32) return set_error(SA_ERR_INVALID_ARG, "dtype must be SA_BF16 or SA_FP32");
  if (nrows < 0 || BH < 0 || N < 1 || dv < 1) return set_error(SA_ERR_INVALID_ARG, "bad sizes for sa_rows_mse");
  if (BH > 2147483647) return set_error(SA_ERR_UNSUPPORTED, "too many heads");
  if (sa_status e = check_device()) return e;
  return launch_rows_mse(ref, x, rows, nrows, BH, N, dv, dtype, out, status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
