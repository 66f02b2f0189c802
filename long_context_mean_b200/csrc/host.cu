// sa_forward_host: the whole forward path from host buffers to host buffers.
//
// The problem is cut into `chunks` groups of (batch, head) rows (whole kv
// groups: query row r reads kv row r / (Hq / Hkv)).  Chunk i's host-to-device
// copies of Q, K, V run on the copy-in stream; its path (layout once, then
// mask prediction fused with the Q/K reorder, the V reorder, block-sparse
// attention with the fused inverse reorder) on the compute stream; its
// device-to-host copies of O and LSE on the copy-out stream.  The copies of
// one chunk overlap the kernels of its neighbours ([P1] section 6: the
// permutation and the data movement count in end-to-end time).  Every device
// buffer comes from the caller's workspace; the call only enqueues.
#include "sa_internal.cuh"

namespace sa {
namespace {

__global__ void status_max_kernel(int32_t* total, const int32_t* part) {
  const int32_t v = *part;
  if (v != 0) atomicMax(total, v);
}

struct HostPlan {
  int64_t rows_q, rows_kv;   // query and kv rows of one chunk
  sa_shape chunk;            // the chunk as a problem of its own: B = 1
  int64_t nqb, nkb, R;
  size_t off[17];            // region offsets in the workspace
  size_t total;
};

enum Region {
  kQ, kK, kV, kOut, kLse, kPerm, kInv, kLayoutWs, kQr, kKr, kVr, kPredWs, kMask, kRowPtr, kColIdx, kOrder,
  kTail   // attention workspace (256 bytes), kept_total (int64), chunk status (int32)
};

size_t region(size_t bytes) { return align_up(bytes ? bytes : 1, 256); }

sa_status plan(const sa_shape& s, const sa_layout_desc& lay, const sa_mask_params& p, int32_t chunks,
               HostPlan& h) {
  if (chunks < 1 || (s.B * s.Hkv) % chunks)
    return set_error(SA_ERR_INVALID_ARG, "chunks must divide B * Hkv (%lld)", (long long)(s.B * s.Hkv));
  if (p.bq < 1 || p.bk < 1) return set_error(SA_ERR_INVALID_ARG, "bq and bk must be positive");
  const int64_t g = s.Hq / s.Hkv;
  h.rows_kv = s.B * s.Hkv / chunks;
  h.rows_q = h.rows_kv * g;
  h.chunk = s;
  h.chunk.B = 1;
  h.chunk.Hq = h.rows_q;
  h.chunk.Hkv = h.rows_kv;
  h.nqb = ceil_div(s.N, p.bq);
  h.nkb = ceil_div(s.N, p.bk);
  h.R = h.rows_q * h.nqb;
  const size_t es = s.dtype == SA_BF16 ? 2 : 4;
  const size_t N = (size_t)s.N;
  const bool reorder = lay.mode != SA_ORDER_IDENTITY;
  const size_t pred = sa_predict_mask_workspace(&h.chunk, &p);
  if (pred == 0) return set_error(SA_ERR_INVALID_ARG, "no mask prediction for this chunk shape: %s", sa_last_error());
  const size_t sizes[17] = {
      (size_t)(s.B * s.Hq) * N * s.d * es,  (size_t)(s.B * s.Hkv) * N * s.d * es,
      (size_t)(s.B * s.Hkv) * N * s.dv * es, (size_t)(s.B * s.Hq) * N * s.dv * es,
      (size_t)(s.B * s.Hq) * N * 4,
      N * 4, N * 4, reorder ? sa_layout_workspace(&lay) : 0,
      reorder ? (size_t)h.rows_q * N * s.d * es : 0, reorder ? (size_t)h.rows_kv * N * s.d * es : 0,
      reorder ? (size_t)h.rows_kv * N * s.dv * es : 0,
      pred,
      (size_t)(h.R * h.nkb), (size_t)(h.R + 1) * 4, (size_t)(h.R * h.nkb) * 4, (size_t)h.R * 4,
      256 + 8 + 8};
  size_t at = 0;
  for (int i = 0; i < 17; ++i) {
    h.off[i] = at;
    at += region(sizes[i]);
  }
  h.total = at;
  return SA_OK;
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" size_t sa_forward_host_workspace(const sa_shape* shape, const sa_layout_desc* layout,
                                            const sa_mask_params* params, int32_t chunks) {
  if (!shape || !layout || !params) return 0;
  HostPlan h;
  if (plan(*shape, *layout, *params, chunks, h) != SA_OK) return 0;
  return h.total;
}

extern "C" sa_status sa_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                     float* lse_host, const sa_shape* shape, const sa_layout_desc* layout,
                                     const sa_mask_params* params, float lambda, float scale, int32_t chunks,
                                     void* ws, size_t ws_bytes, int32_t* status, void* const streams[3]) {
  if (!q_host || !k_host || !v_host || !out_host || !lse_host || !shape || !layout || !params || !status ||
      !streams)
    return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_forward_host");
  if (shape->N != layout->T * layout->H * layout->W + layout->txt_len)
    return set_error(SA_ERR_INVALID_ARG, "shape N differs from the layout's token count");
  HostPlan h;
  if (sa_status e = plan(*shape, *layout, *params, chunks, h)) return e;
  if (!ws || ws_bytes < h.total || (uintptr_t)ws % 256)
    return set_error(SA_ERR_WORKSPACE, "sa_forward_host needs %zu bytes of 256-byte aligned workspace", h.total);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return set_error(SA_ERR_CUDA, "no usable CUDA device");
  }
  cudaStream_t comp = static_cast<cudaStream_t>(streams[0]);
  cudaStream_t s_in = static_cast<cudaStream_t>(streams[1]);
  cudaStream_t s_out = static_cast<cudaStream_t>(streams[2]);
  char* base = static_cast<char*>(ws);
  auto at = [&](int r) { return base + h.off[r]; };
  const sa_shape& s = *shape;
  const size_t es = s.dtype == SA_BF16 ? 2 : 4;
  const size_t qrow = (size_t)s.N * s.d * es, vrow = (size_t)s.N * s.dv * es, orow = (size_t)s.N * s.dv * es;
  const bool reorder = layout->mode != SA_ORDER_IDENTITY;
  int32_t* perm = reinterpret_cast<int32_t*>(at(kPerm));
  int32_t* inv = reinterpret_cast<int32_t*>(at(kInv));
  char* tail = at(kTail);
  sa_mask m{};
  m.block_mask = reinterpret_cast<uint8_t*>(at(kMask));
  m.row_ptr = reinterpret_cast<int32_t*>(at(kRowPtr));
  m.col_idx = reinterpret_cast<int32_t*>(at(kColIdx));
  m.order = reinterpret_cast<int32_t*>(at(kOrder));
  void* attn_ws = tail;   // 256-byte aligned, as every region
  m.kept_total = reinterpret_cast<int64_t*>(tail + 256);
  m.status = reinterpret_cast<int32_t*>(tail + 264);
  m.col_capacity = h.R * h.nkb;
  const size_t pred_bytes = h.off[kPredWs + 1] - h.off[kPredWs];

  // Events ordering the three streams (released once their work completes).
  const int nev = 3 * chunks + 1;
  cudaEvent_t ev_small[3 * 16 + 1];
  cudaEvent_t* ev = ev_small;
  if (nev > 3 * 16 + 1) return set_error(SA_ERR_UNSUPPORTED, "at most 16 chunks");
  int made = 0;
  sa_status rc = SA_OK;
  for (; made < nev; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) {
      rc = set_error(SA_ERR_CUDA, "cudaEventCreate failed");
      break;
    }
  cudaEvent_t start = ev[0];
  auto e_in = [&](int i) { return ev[1 + 3 * i]; };
  auto e_comp = [&](int i) { return ev[2 + 3 * i]; };
  auto e_out = [&](int i) { return ev[3 + 3 * i]; };
  auto cuda_ok = [&](cudaError_t e, const char* what) {
    if (e != cudaSuccess && rc == SA_OK) rc = set_error(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return rc == SA_OK;
  };
  if (rc == SA_OK && cuda_ok(cudaMemsetAsync(status, 0, sizeof(int32_t), comp), "cudaMemsetAsync(status)") &&
      cuda_ok(cudaEventRecord(start, comp), "cudaEventRecord")) {
    if (reorder) {
      const size_t lws = h.off[kLayoutWs + 1] - h.off[kLayoutWs];
      rc = sa_layout_build(layout, perm, inv, lws ? at(kLayoutWs) : nullptr, lws, comp);
    }
    for (int i = 0; i < chunks && rc == SA_OK; ++i) {
      const size_t qo = (size_t)(i * h.rows_q) * qrow, ko = (size_t)(i * h.rows_kv) * qrow;
      const size_t vo = (size_t)(i * h.rows_kv) * vrow, oo = (size_t)(i * h.rows_q) * orow;
      const size_t lo = (size_t)(i * h.rows_q) * s.N * 4;
      char* qd = at(kQ) + qo;
      char* kd = at(kK) + ko;
      char* vd = at(kV) + vo;
      char* od = at(kOut) + oo;
      float* ld = reinterpret_cast<float*>(at(kLse) + lo);
      // host -> device, after everything the caller enqueued on the compute stream
      if (!cuda_ok(cudaStreamWaitEvent(s_in, start, 0), "cudaStreamWaitEvent") ||
          !cuda_ok(cudaMemcpyAsync(qd, static_cast<const char*>(q_host) + qo, h.rows_q * qrow,
                                   cudaMemcpyHostToDevice, s_in), "cudaMemcpyAsync(q)") ||
          !cuda_ok(cudaMemcpyAsync(kd, static_cast<const char*>(k_host) + ko, h.rows_kv * qrow,
                                   cudaMemcpyHostToDevice, s_in), "cudaMemcpyAsync(k)") ||
          !cuda_ok(cudaMemcpyAsync(vd, static_cast<const char*>(v_host) + vo, h.rows_kv * vrow,
                                   cudaMemcpyHostToDevice, s_in), "cudaMemcpyAsync(v)") ||
          !cuda_ok(cudaEventRecord(e_in(i), s_in), "cudaEventRecord") ||
          !cuda_ok(cudaStreamWaitEvent(comp, e_in(i), 0), "cudaStreamWaitEvent"))
        break;
      // the path on this chunk
      const void *qa = qd, *ka = kd, *va = vd;
      if (reorder) {
        if ((rc = sa_reorder_predict_mask(perm, qd, kd, at(kQr), at(kKr), &h.chunk, params, at(kPredWs),
                                          pred_bytes, &m, comp)))
          break;
        if ((rc = sa_reorder(perm, vd, at(kVr), h.rows_kv, s.N, s.dv, s.dtype, comp))) break;
        qa = at(kQr);
        ka = at(kKr);
        va = at(kVr);
      } else if ((rc = sa_predict_mask(qd, kd, &h.chunk, params, at(kPredWs), pred_bytes, &m, comp))) {
        break;
      }
      if ((rc = sa_block_sparse_attn(qa, ka, va, &h.chunk, &m, lambda, scale, od, ld, reorder ? perm : nullptr,
                                     nullptr, attn_ws, 256, 0, comp)))
        break;
      status_max_kernel<<<1, 1, 0, comp>>>(status, m.status);
      if ((rc = check_launch("status_max_kernel"))) break;
      // device -> host
      if (!cuda_ok(cudaEventRecord(e_comp(i), comp), "cudaEventRecord") ||
          !cuda_ok(cudaStreamWaitEvent(s_out, e_comp(i), 0), "cudaStreamWaitEvent") ||
          !cuda_ok(cudaMemcpyAsync(static_cast<char*>(out_host) + oo, od, h.rows_q * orow, cudaMemcpyDeviceToHost,
                                   s_out), "cudaMemcpyAsync(out)") ||
          !cuda_ok(cudaMemcpyAsync(reinterpret_cast<char*>(lse_host) + lo, ld, (size_t)h.rows_q * s.N * 4,
                                   cudaMemcpyDeviceToHost, s_out), "cudaMemcpyAsync(lse)") ||
          !cuda_ok(cudaEventRecord(e_out(i), s_out), "cudaEventRecord"))
        break;
    }
    // The call is complete on the compute stream once the last copy back is.
    if (rc == SA_OK) cuda_ok(cudaStreamWaitEvent(comp, e_out(chunks - 1), 0), "cudaStreamWaitEvent");
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  return rc;
}
