// extern "C" entry points of libegat.so: argument validation, workspace
// carving and dispatch to the kernels.  The ABI itself is documented in
// include/egat.h.
#include <cstring>

#include "egat_device.cuh"
#include "egat_host.h"

using namespace egat;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Shape checks common to steps 2-4 (supported set stated in egat.h).
int check_shape(const egat_shape* s, bool need_graph) {
  if (!s) return EGAT_ERR_ARG;
  if (s->n < 0) return EGAT_ERR_ARG;
  if (s->dtype != EGAT_F32 && s->dtype != EGAT_BF16) return EGAT_ERR_ARG;
  if (s->lmax < 1 || s->lmax > kMaxL) return EGAT_ERR_UNSUPPORTED;
  if (s->C != 16 && s->C != 32 && s->C != 64 && s->C != 128) return EGAT_ERR_UNSUPPORTED;
  if (need_graph) {
    if (!pow2(s->H) || s->C % s->H != 0 || (s->C / s->H) % 8 != 0) return EGAT_ERR_UNSUPPORTED;
    if (s->dk != 8 && s->dk != 16 && s->dk != 32) return EGAT_ERR_UNSUPPORTED;
    if (s->H * s->dk > 256) return EGAT_ERR_UNSUPPORTED;
    if (s->graph_mode == EGAT_GRAPH_PADDED) {
      if (s->K < 1 || s->K > 1024) return EGAT_ERR_ARG;
    } else if (s->graph_mode == EGAT_GRAPH_CSR) {
      if (s->n_edges < 0) return EGAT_ERR_ARG;
    } else {
      return EGAT_ERR_ARG;
    }
  }
  return EGAT_OK;
}

size_t hp_bytes(const egat_shape& s) {
  const size_t D = size_t(s.lmax + 1) * (s.lmax + 1);
  return (size_t(s.n) * D * s.C * storage_bytes(s.dtype) + 255) & ~size_t(255);
}

// forward workspace: h', then (tensor-core shapes) the attention plan
size_t forward_ws_bytes(const egat_shape& s) {
  size_t b = hp_bytes(s);
  if (tc_attention_supported(s) && s.n > 0) b += plan_bytes(s.n, s.K, s.lmax);
  return b;
}

}  // namespace

extern "C" {

int egat_version(void) { return EGAT_VERSION; }

const char* egat_strerror(int code) {
  switch (code) {
    case EGAT_OK: return "success";
    case EGAT_ERR_ARG: return "invalid argument (null pointer, size or alignment)";
    case EGAT_ERR_UNSUPPORTED: return "shape outside the supported set";
    case EGAT_ERR_CUDA: return "CUDA launch or runtime error";
    case EGAT_ERR_WORKSPACE: return "workspace too small";
    case EGAT_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than egat_forward_noalloc's fixed array holds";
    case EGAT_ERR_TIMEOUT: return "a bounded device wait gave up (results of that launch are invalid)";
    default: return "unknown egat status";
  }
}

int egat_num_paths(int lmax) {
  if (lmax < 0 || lmax > kMaxL) return 0;
  return num_paths(lmax);
}

int egat_graph_workspace_bytes(int32_t n, size_t* bytes) {
  if (!bytes || n < 0) return EGAT_ERR_ARG;
  *bytes = graph_workspace_bytes(n);
  return EGAT_OK;
}

int egat_build_graph(const int32_t* d_pos_q, int32_t n, int32_t cutoff_q, int32_t K, int32_t mode,
                     int32_t* d_nbr_or_rowptr, int32_t* d_cnt_or_col, int64_t col_capacity,
                     int32_t* d_order, int32_t* d_overflow, void* d_ws, size_t ws_bytes,
                     void* stream) {
  if (n < 0 || cutoff_q <= 0 || !d_overflow) return EGAT_ERR_ARG;
  // candidate cells span at most 20 cells of edge ceil(cutoff_q / 2) per axis;
  // this keeps every coordinate difference the kernels form within 32 bits
  if (cutoff_q > (1 << 26)) return EGAT_ERR_UNSUPPORTED;
  if (mode == EGAT_GRAPH_PADDED) {
    if (K < 1 || K > 1024) return EGAT_ERR_ARG;
  } else if (mode == EGAT_GRAPH_CSR) {
    if (col_capacity < 0) return EGAT_ERR_ARG;
  } else {
    return EGAT_ERR_ARG;
  }
  // keys are (d^2 << ceil(log2 n)) | j in 64 bits
  int shift = 1;
  while ((int64_t(1) << shift) < int64_t(n)) ++shift;
  const unsigned __int128 top = (unsigned __int128)((uint64_t)cutoff_q * (uint64_t)cutoff_q) << shift;
  if (top >> 64) return EGAT_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n == 0) {
    if (mode == EGAT_GRAPH_CSR && d_nbr_or_rowptr &&
        cudaMemsetAsync(d_nbr_or_rowptr, 0, sizeof(int32_t), st) != cudaSuccess)
      return EGAT_ERR_CUDA;
    return cudaMemsetAsync(d_overflow, 0, sizeof(int32_t), st) == cudaSuccess ? EGAT_OK
                                                                              : EGAT_ERR_CUDA;
  }
  if (!d_pos_q || !d_nbr_or_rowptr || !d_ws) return EGAT_ERR_ARG;
  if (!d_cnt_or_col && !(mode == EGAT_GRAPH_CSR && col_capacity == 0)) return EGAT_ERR_ARG;
  if (!aligned4(d_pos_q) || !aligned4(d_nbr_or_rowptr) || !aligned4(d_overflow)) return EGAT_ERR_ARG;
  if (!aligned16(d_ws)) return EGAT_ERR_ARG;
  return build_graph(d_pos_q, n, cutoff_q, K, mode, d_nbr_or_rowptr, d_cnt_or_col, col_capacity,
                     d_order, d_overflow, d_ws, ws_bytes, st);
}

int egat_eaas_couple(const egat_shape* s, const void* d_x, const float* d_pos, const float* d_w,
                     void* d_y, void* stream) {
  const int rc = check_shape(s, false);
  if (rc != EGAT_OK) return rc;
  if (s->n == 0) return EGAT_OK;
  if (!d_x || !d_pos || !d_w || !d_y) return EGAT_ERR_ARG;
  if (!aligned16(d_x) || !aligned16(d_y) || !aligned4(d_pos) || !aligned4(d_w)) return EGAT_ERR_ARG;
  return launch_eaas_source(*s, d_x, d_pos, d_w, d_y, static_cast<cudaStream_t>(stream));
}

int egat_otf_attention(const egat_shape* s, const void* d_q, const void* d_k, const void* d_hp,
                       const int32_t* d_nbr_or_rowptr, const int32_t* d_cnt_or_col,
                       const int32_t* d_order, float* d_m, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->n == 0) return EGAT_OK;
  if (!d_q || !d_k || !d_hp || !d_nbr_or_rowptr || !d_m) return EGAT_ERR_ARG;
  if (s->graph_mode == EGAT_GRAPH_CSR && !d_cnt_or_col && s->n_edges > 0) return EGAT_ERR_ARG;
  if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_hp) || !aligned16(d_m)) return EGAT_ERR_ARG;
  return launch_attention(*s, false, d_q, d_k, d_hp, d_nbr_or_rowptr, d_cnt_or_col, d_order,
                          nullptr, nullptr, d_m, static_cast<cudaStream_t>(stream));
}

int egat_otf_attention_coupled(const egat_shape* s, const void* d_q, const void* d_k,
                               const void* d_hp, const int32_t* d_nbr_or_rowptr,
                               const int32_t* d_cnt_or_col, const int32_t* d_order,
                               const float* d_pos, const float* d_w2, float* d_out, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->n == 0) return EGAT_OK;
  if (!d_q || !d_k || !d_hp || !d_nbr_or_rowptr || !d_pos || !d_w2 || !d_out) return EGAT_ERR_ARG;
  if (s->graph_mode == EGAT_GRAPH_CSR && !d_cnt_or_col && s->n_edges > 0) return EGAT_ERR_ARG;
  if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_hp) || !aligned16(d_out) ||
      !aligned4(d_pos) || !aligned4(d_w2))
    return EGAT_ERR_ARG;
  return launch_attention(*s, true, d_q, d_k, d_hp, d_nbr_or_rowptr, d_cnt_or_col, d_order, d_pos,
                          d_w2, d_out, static_cast<cudaStream_t>(stream));
}

int egat_forward_workspace_bytes(const egat_shape* s, size_t* bytes) {
  if (!bytes) return EGAT_ERR_ARG;
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  *bytes = forward_ws_bytes(*s);
  return EGAT_OK;
}

int egat_attention_plan_bytes(const egat_shape* s, size_t* bytes) {
  if (!bytes) return EGAT_ERR_ARG;
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if (plan_smem_bytes(s->n, s->K) > kPlanSmemLimit) return EGAT_ERR_UNSUPPORTED;
  *bytes = s->n > 0 ? plan_bytes(s->n, s->K, s->lmax) : 0;
  return EGAT_OK;
}

int egat_build_attention_plan(const egat_shape* s, const int32_t* d_nbr, const int32_t* d_cnt,
                              const int32_t* d_order, const float* d_pos, void* d_plan,
                              size_t plan_bytes_given, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if (plan_smem_bytes(s->n, s->K) > kPlanSmemLimit) return EGAT_ERR_UNSUPPORTED;
  if (s->n == 0) return EGAT_OK;
  if (!d_nbr || !d_pos || !d_plan) return EGAT_ERR_ARG;
  if (!aligned16(d_plan) || !aligned4(d_nbr) || !aligned4(d_pos)) return EGAT_ERR_ARG;
  if (plan_bytes_given < plan_bytes(s->n, s->K, s->lmax)) return EGAT_ERR_WORKSPACE;
  return launch_build_plan(s->n, s->K, s->lmax, d_nbr, d_cnt, d_order, d_pos, d_plan,
                           static_cast<cudaStream_t>(stream));
}

int egat_eaas_couple_planned(const egat_shape* s, const void* d_h, const void* d_plan,
                             const float* d_w1, void* d_hout, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if (plan_smem_bytes(s->n, s->K) > kPlanSmemLimit) return EGAT_ERR_UNSUPPORTED;
  if (s->n == 0) return EGAT_OK;
  if (!d_h || !d_plan || !d_w1 || !d_hout) return EGAT_ERR_ARG;
  if (!aligned16(d_h) || !aligned16(d_plan) || !aligned16(d_hout) || !aligned4(d_w1))
    return EGAT_ERR_ARG;
  return launch_eaas_planned(*s, d_h, d_plan, d_w1, d_hout, static_cast<cudaStream_t>(stream));
}

int egat_otf_attention_tiled(const egat_shape* s, const void* d_q, const void* d_k,
                             const void* d_hp, const void* d_plan, const float* d_w2,
                             float* d_out, int32_t fused, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (!tc_attention_supported(*s)) return EGAT_ERR_UNSUPPORTED;
  if (s->n == 0) return EGAT_OK;
  if (!d_q || !d_k || !d_hp || !d_plan || !d_out) return EGAT_ERR_ARG;
  if (fused && !d_w2) return EGAT_ERR_ARG;
  if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_hp) || !aligned16(d_plan) ||
      !aligned16(d_out))
    return EGAT_ERR_ARG;
  if (fused && !aligned4(d_w2)) return EGAT_ERR_ARG;
  return launch_attention_tc(*s, fused != 0, d_q, d_k, d_hp, d_plan, d_w2, d_out,
                             static_cast<cudaStream_t>(stream));
}

int egat_forward(const egat_shape* s, const void* d_h, const float* d_pos, const void* d_q,
                 const void* d_k, const int32_t* d_nbr_or_rowptr, const int32_t* d_cnt_or_col,
                 const int32_t* d_order, const float* d_w1, const float* d_w2, void* d_ws,
                 size_t ws_bytes, float* d_out, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->n == 0) return EGAT_OK;
  if (!d_h || !d_pos || !d_q || !d_k || !d_nbr_or_rowptr || !d_w1 || !d_w2 || !d_ws || !d_out)
    return EGAT_ERR_ARG;
  if (s->graph_mode == EGAT_GRAPH_CSR && !d_cnt_or_col && s->n_edges > 0) return EGAT_ERR_ARG;
  if (!aligned16(d_h) || !aligned16(d_q) || !aligned16(d_k) || !aligned16(d_ws) ||
      !aligned16(d_out) || !aligned4(d_pos) || !aligned4(d_w1) || !aligned4(d_w2))
    return EGAT_ERR_ARG;
  if (ws_bytes < forward_ws_bytes(*s)) return EGAT_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_attention_supported(*s)) {
    void* plan = static_cast<char*>(d_ws) + hp_bytes(*s);
    int e = launch_build_plan(s->n, s->K, s->lmax, d_nbr_or_rowptr, d_cnt_or_col, d_order, d_pos,
                              plan, st);
    if (e != EGAT_OK) return e;
    e = launch_eaas_planned(*s, d_h, plan, d_w1, d_ws, st);
    if (e != EGAT_OK) return e;
    return launch_attention_tc(*s, true, d_q, d_k, d_ws, plan, d_w2, d_out, st);
  }
  int e = launch_eaas_source(*s, d_h, d_pos, d_w1, d_ws, st);
  if (e != EGAT_OK) return e;
  return launch_attention(*s, true, d_q, d_k, d_ws, d_nbr_or_rowptr, d_cnt_or_col, d_order, d_pos,
                          d_w2, d_out, st);
}

}  // extern "C"

int egat_take_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int a = 0, b = 0, c = 0, d = 0;
  const int ra = take_wait_timeouts_attention(st, &a);
  const int rb = take_wait_timeouts_coupling(st, &b);
  const int rc = take_wait_timeouts_backward(st, &c);
  const int rd = take_wait_timeouts_projection(st, &d);
  if (ra != EGAT_OK) return ra;
  if (rb != EGAT_OK) return rb;
  if (rc != EGAT_OK) return rc;
  if (rd != EGAT_OK) return rd;
  return (a | b | c | d) ? EGAT_ERR_TIMEOUT : EGAT_OK;
}

int egat_qk_projection(const egat_shape* s, const void* d_h, const float* d_wq, const float* d_wk,
                       void* d_q, void* d_k, void* stream) {
  if (!s || s->n < 0) return EGAT_ERR_ARG;
  if (s->dtype != EGAT_F32 && s->dtype != EGAT_BF16) return EGAT_ERR_ARG;
  if (s->lmax < 0 || s->lmax > kMaxL) return EGAT_ERR_UNSUPPORTED;
  if (s->C < 1 || s->C > 1024 || s->H < 1 || s->dk < 1 || s->H * s->dk > 1024)
    return EGAT_ERR_UNSUPPORTED;
  if (s->n == 0) return EGAT_OK;
  if (!d_h || !d_wq || !d_wk || !d_q || !d_k) return EGAT_ERR_ARG;
  if (!aligned16(d_h) || !aligned4(d_wq) || !aligned4(d_wk) || !aligned4(d_q) || !aligned4(d_k))
    return EGAT_ERR_ARG;
  return launch_qk_projection(*s, d_h, d_wq, d_wk, d_q, d_k, static_cast<cudaStream_t>(stream));
}

int egat_escn_num_weights(int32_t lmax, int32_t mmax) {
  if (lmax < 1 || lmax > kMaxL || mmax < 0 || mmax > lmax) return 0;
  return escn_num_weights_host(lmax, mmax);
}

int egat_escn_conv(const egat_shape* s, int32_t mmax, const void* d_h, const float* d_pos,
                   const int32_t* d_nbr, const int32_t* d_cnt, const int32_t* d_order,
                   const float* d_w, float* d_out, void* stream) {
  const int rc = check_shape(s, false);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if (s->K < 1 || s->K > 1024) return EGAT_ERR_ARG;
  if (mmax < 0 || mmax > s->lmax) return EGAT_ERR_ARG;
  if (s->n == 0) return EGAT_OK;
  if (!d_h || !d_pos || !d_nbr || !d_w || !d_out) return EGAT_ERR_ARG;
  if (!aligned16(d_h) || !aligned4(d_pos) || !aligned4(d_nbr) || !aligned4(d_w) ||
      !aligned4(d_out) || (d_cnt && !aligned4(d_cnt)) || (d_order && !aligned4(d_order)))
    return EGAT_ERR_ARG;
  return launch_escn_conv(*s, mmax, d_h, d_pos, d_nbr, d_cnt, d_order, d_w, d_out,
                          static_cast<cudaStream_t>(stream));
}

int egat_gather_rows(const void* d_src, int64_t n_src, int64_t row_bytes, const int32_t* d_idx,
                     int64_t count, void* d_dst, void* stream) {
  if (n_src < 0 || count < 0 || row_bytes <= 0 || row_bytes % 16) return EGAT_ERR_ARG;
  if (count == 0) return EGAT_OK;
  if (!d_idx || !d_dst || (n_src > 0 && !d_src)) return EGAT_ERR_ARG;
  if (!aligned16(d_dst) || (d_src && !aligned16(d_src)) || !aligned4(d_idx)) return EGAT_ERR_ARG;
  return launch_gather_rows(d_src, n_src, row_bytes, d_idx, count, d_dst,
                            static_cast<cudaStream_t>(stream));
}

int egat_selftest_wait_timeout(int32_t polls, void* stream) {
  if (polls < 1 || polls > (1 << 20)) return EGAT_ERR_ARG;
  return launch_wait_timeout_selftest(polls, static_cast<cudaStream_t>(stream));
}

int egat_backward_workspace_bytes(const egat_shape* s, size_t* bytes) {
  if (!bytes) return EGAT_ERR_ARG;
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if ((long long)s->n * s->K >= (1LL << 31)) return EGAT_ERR_UNSUPPORTED;
  *bytes = s->n > 0 ? backward_ws_bytes(*s) : 0;
  return EGAT_OK;
}

int egat_backward(const egat_shape* s, const void* d_h, const float* d_pos, const void* d_q,
                  const void* d_k, const int32_t* d_nbr, const int32_t* d_cnt,
                  const int32_t* d_order, const float* d_w1, const float* d_w2,
                  const float* d_grad_out, void* d_ws, size_t ws_bytes, float* d_dh, float* d_dq,
                  float* d_dk, float* d_dpos, void* stream) {
  const int rc = check_shape(s, true);
  if (rc != EGAT_OK) return rc;
  if (s->graph_mode != EGAT_GRAPH_PADDED) return EGAT_ERR_UNSUPPORTED;
  if ((long long)s->n * s->K >= (1LL << 31)) return EGAT_ERR_UNSUPPORTED;
  if (s->n == 0) return EGAT_OK;
  if (!d_h || !d_pos || !d_q || !d_k || !d_nbr || !d_w1 || !d_w2 || !d_grad_out || !d_ws ||
      !d_dh || !d_dq || !d_dk)
    return EGAT_ERR_ARG;
  if (!aligned16(d_h) || !aligned16(d_q) || !aligned16(d_k) || !aligned16(d_ws) ||
      !aligned16(d_grad_out) || !aligned16(d_dh) || !aligned16(d_dq) || !aligned16(d_dk) ||
      !aligned4(d_pos) || !aligned4(d_nbr) || !aligned4(d_w1) || !aligned4(d_w2) ||
      (d_dpos && !aligned4(d_dpos)) || (d_order && !aligned4(d_order)))
    return EGAT_ERR_ARG;
  if (ws_bytes < backward_ws_bytes(*s)) return EGAT_ERR_WORKSPACE;
  return launch_backward(*s, d_h, d_pos, d_q, d_k, d_nbr, d_cnt, d_order, d_w1, d_w2, d_grad_out,
                         d_ws, d_dh, d_dq, d_dk, d_dpos, static_cast<cudaStream_t>(stream));
}
