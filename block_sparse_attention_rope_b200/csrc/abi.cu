// abi.cu -- argument checking and dispatch of the attention entry points,
// the per-device status word, status strings.
#include <mutex>

#include "lc_internal.cuh"

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int *g_status[kMaxDevices] = {nullptr};

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// A shard plan is accepted by lc_bsa_forward_shard only (allow_shard).
lc_status check_common(const lc_bsa_plan_s *plan, const lc_rope3d_s *rope, int batch, int heads,
                       int head_dim, lc_dtype dtype, bool allow_shard = false) {
  if (!plan || !rope || batch <= 0 || heads <= 0 || head_dim <= 0)
    return LC_ERR_INVALID_ARGUMENT;
  if (!allow_shard && lc_plan_is_shard(plan)) return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16 && dtype != LC_DTYPE_F32) return LC_ERR_INVALID_ARGUMENT;
  if (head_dim != LC_HEAD_DIM) return LC_ERR_UNSUPPORTED;
  if (plan->T != rope->T || plan->H != rope->H || plan->W != rope->W)
    return LC_ERR_INVALID_ARGUMENT;
  long long rows = (long long)batch * (plan->Nc + plan->Nn) * heads;
  if (rows * LC_HEAD_DIM >= (1LL << 40)) return LC_ERR_UNSUPPORTED;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return LC_ERR_CUDA;
  if (dev != plan->device || dev != rope->device) return LC_ERR_INVALID_ARGUMENT;
  return LC_OK;
}

lc_status run_forward(const void *q, const void *k, const void *v, const void *cond_k,
                      const void *cond_v, void *out, float *lse, int batch, int heads, int head_dim,
                      lc_dtype dtype, float softmax_scale, lc_bsa_plan plan, lc_rope3d rope,
                      void *stream, lc_fwd_mode mode, bool cond_k_rotated,
                      const lc_qk_norm &norm = lc_qk_norm()) {
  lc_status s = check_common(plan, rope, batch, heads, head_dim, dtype);
  if (s != LC_OK) return s;
  const bool cond_only = mode == LC_FWD_COND, split = mode != LC_FWD_FULL;
  if (!q || !out || (!cond_only && (!k || !v))) return LC_ERR_INVALID_ARGUMENT;
  if (split && plan->Nc > 0 && (!cond_k || !cond_v)) return LC_ERR_INVALID_ARGUMENT;
  if (misaligned(q) || misaligned(out) || (!cond_only && (misaligned(k) || misaligned(v))) ||
      (split && plan->Nc > 0 && (misaligned(cond_k) || misaligned(cond_v))) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return LC_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale)) return LC_ERR_INVALID_ARGUMENT;  // NaN
  float scale = softmax_scale > 0.f ? softmax_scale : 0.125f;  // 1/sqrt(64)
  int *dev_status = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == LC_DTYPE_F32)
    return lc_launch_forward_f32(static_cast<const float *>(q), static_cast<const float *>(k),
                                 static_cast<const float *>(v), static_cast<const float *>(cond_k),
                                 static_cast<const float *>(cond_v), static_cast<float *>(out),
                                 lse, batch, heads, scale, mode, cond_k_rotated, norm, plan,
                                 rope, dev_status, st);
  return lc_launch_forward_sm100(q, k, v, cond_k, cond_v, out, lse, batch, heads, scale, mode,
                                 cond_k_rotated, norm, plan, rope, dev_status, st);
}

// Options -> flags and norm; false on a bad option.
bool parse_opts(const lc_bsa_opts *opts, unsigned allowed_flags, unsigned *flags,
                lc_qk_norm *norm) {
  *flags = 0;
  *norm = lc_qk_norm();
  if (!opts) return true;
  if (opts->flags & ~allowed_flags) return false;
  *flags = opts->flags;
  const bool any = opts->q_norm_weight || opts->k_norm_weight;
  if (any && !(opts->norm_eps >= 0.f && opts->norm_eps <= 3.0e38f)) return false;  // NaN, inf
  if ((reinterpret_cast<uintptr_t>(opts->q_norm_weight) |
       reinterpret_cast<uintptr_t>(opts->k_norm_weight)) & 3u)
    return false;
  norm->q_w = opts->q_norm_weight;
  norm->k_w = opts->k_norm_weight;
  norm->eps = opts->norm_eps;
  return true;
}

}  // namespace

namespace {
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxDevices] = {nullptr};
}  // namespace

// The library's own stream-ordered pool for per-call scratch.  It keeps what
// it has allocated (release threshold = all), so steady-state calls reuse the
// memory with no driver allocation, and the device's default pool is left
// untouched.  The memory stays with the process until it exits.
cudaMemPool_t lc_scratch_pool(lc_status *st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = LC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    e = cudaMemPoolCreate(&pool, &props);
    if (e == cudaSuccess) {
      uint64_t keep = ~0ull;
      e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    }
    if (e != cudaSuccess) {
      *st = lc_from_cuda(e);
      return nullptr;
    }
    g_pool[dev] = pool;
  }
  *st = LC_OK;
  return g_pool[dev];
}

int *lc_device_status_ptr(lc_status *st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = LC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status[dev]) {
    int *p = nullptr;
    e = cudaMalloc(&p, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(int));
    if (e != cudaSuccess) {
      *st = lc_from_cuda(e);
      return nullptr;
    }
    g_status[dev] = p;
  }
  *st = LC_OK;
  return g_status[dev];
}

extern "C" lc_status lc_bsa_forward(const void *q, const void *k, const void *v, void *out,
                                    float *lse, int batch, int heads, int head_dim, lc_dtype dtype,
                                    float softmax_scale, lc_bsa_plan plan, lc_rope3d rope,
                                    void *stream) {
  return run_forward(q, k, v, nullptr, nullptr, out, lse, batch, heads, head_dim, dtype,
                     softmax_scale, plan, rope, stream, LC_FWD_FULL, false);
}

extern "C" lc_status lc_bsa_forward_cached(const void *q, const void *k, const void *v,
                                           const void *cond_k, const void *cond_v, void *out,
                                           float *lse, int batch, int heads, int head_dim,
                                           lc_dtype dtype, float softmax_scale, lc_bsa_plan plan,
                                           lc_rope3d rope, void *stream) {
  return run_forward(q, k, v, cond_k, cond_v, out, lse, batch, heads, head_dim, dtype,
                     softmax_scale, plan, rope, stream, LC_FWD_CACHED, false);
}

extern "C" lc_status lc_bsa_forward_ex(const void *q, const void *k, const void *v, void *out,
                                       float *lse, int batch, int heads, int head_dim,
                                       lc_dtype dtype, float softmax_scale,
                                       const lc_bsa_opts *opts, lc_bsa_plan plan, lc_rope3d rope,
                                       void *stream) {
  unsigned flags;
  lc_qk_norm norm;
  if (!parse_opts(opts, 0u, &flags, &norm)) return LC_ERR_INVALID_ARGUMENT;
  return run_forward(q, k, v, nullptr, nullptr, out, lse, batch, heads, head_dim, dtype,
                     softmax_scale, plan, rope, stream, LC_FWD_FULL, false, norm);
}

extern "C" lc_status lc_bsa_forward_cached_ex(const void *q, const void *k, const void *v,
                                              const void *cond_k, const void *cond_v, void *out,
                                              float *lse, int batch, int heads, int head_dim,
                                              lc_dtype dtype, float softmax_scale,
                                              const lc_bsa_opts *opts, lc_bsa_plan plan,
                                              lc_rope3d rope, void *stream) {
  unsigned flags;
  lc_qk_norm norm;
  if (!parse_opts(opts, LC_FLAG_COND_K_ROTATED, &flags, &norm)) return LC_ERR_INVALID_ARGUMENT;
  return run_forward(q, k, v, cond_k, cond_v, out, lse, batch, heads, head_dim, dtype,
                     softmax_scale, plan, rope, stream, LC_FWD_CACHED,
                     (flags & LC_FLAG_COND_K_ROTATED) != 0, norm);
}

extern "C" lc_status lc_bsa_backward(const void *q, const void *k, const void *v, const void *out,
                                     const float *lse, const void *dout, void *dq, void *dk,
                                     void *dv, int batch, int heads, int head_dim, lc_dtype dtype,
                                     float softmax_scale, const lc_bsa_opts *opts,
                                     lc_bsa_plan plan, lc_rope3d rope, void *stream) {
  lc_status s = check_common(plan, rope, batch, heads, head_dim, dtype);
  if (s != LC_OK) return s;
  unsigned flags;
  lc_qk_norm norm;
  if (!parse_opts(opts, 0u, &flags, &norm)) return LC_ERR_INVALID_ARGUMENT;
  const void *ins[6] = {q, k, v, out, dout, lse};
  for (const void *p : ins)
    if (!p || misaligned(p)) return LC_ERR_INVALID_ARGUMENT;
  void *outs[3] = {dq, dk, dv};
  for (void *p : outs)
    if (!p || misaligned(p)) return LC_ERR_INVALID_ARGUMENT;
  if (batch > 65535 || heads > 65535) return LC_ERR_UNSUPPORTED;  // grid y / z
  if (!(softmax_scale == softmax_scale)) return LC_ERR_INVALID_ARGUMENT;
  float scale = softmax_scale > 0.f ? softmax_scale : 0.125f;
  return lc_launch_backward(q, k, v, out, lse, dout, dq, dk, dv, batch, heads, scale, dtype, norm,
                            plan, rope, static_cast<cudaStream_t>(stream));
}

extern "C" lc_status lc_bsa_cond_cache(const void *cond_q, const void *cond_k, const void *cond_v,
                                       void *cond_k_rot, void *cond_out, float *cond_lse,
                                       int batch, int heads, int head_dim, lc_dtype dtype,
                                       float softmax_scale, const lc_bsa_opts *opts,
                                       lc_bsa_plan plan, lc_rope3d rope, void *stream) {
  lc_status s = check_common(plan, rope, batch, heads, head_dim, dtype);
  if (s != LC_OK) return s;
  unsigned flags;
  lc_qk_norm norm;
  if (!parse_opts(opts, 0u, &flags, &norm)) return LC_ERR_INVALID_ARGUMENT;
  if (plan->Nc == 0) return LC_OK;
  if (!cond_k || !cond_k_rot || misaligned(cond_k) || misaligned(cond_k_rot))
    return LC_ERR_INVALID_ARGUMENT;
  const size_t elem = dtype == LC_DTYPE_F32 ? 4 : 2;
  const uintptr_t bytes = (uintptr_t)batch * plan->Nc * heads * LC_HEAD_DIM * elem;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(cond_k), b0 = reinterpret_cast<uintptr_t>(cond_k_rot);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return LC_ERR_INVALID_ARGUMENT;  // overlap
  if (cond_out && (!cond_q || !cond_v)) return LC_ERR_INVALID_ARGUMENT;
  if (!cond_out && cond_lse) return LC_ERR_INVALID_ARGUMENT;
  if (cond_out && !(softmax_scale == softmax_scale)) return LC_ERR_INVALID_ARGUMENT;
  // R(norm_k(cond_k)): the same per-row arithmetic as every rotation in the
  // library.
  s = lc_rotate_rows(cond_k, cond_k_rot, batch, plan->Nc, heads, 0, dtype, rope, norm.k_w,
                     norm.eps, static_cast<cudaStream_t>(stream));
  if (s != LC_OK || !cond_out) return s;
  return run_forward(cond_q, nullptr, nullptr, cond_k_rot, cond_v, cond_out, cond_lse, batch,
                     heads, head_dim, dtype, softmax_scale, plan, rope, stream, LC_FWD_COND, true,
                     norm);
}

extern "C" lc_status lc_bsa_forward_noalloc(const void *q, const void *k, const void *v,
                                            void *out, float *lse, int batch, int heads,
                                            int head_dim, lc_dtype dtype, float softmax_scale,
                                            lc_bsa_plan plan, lc_rope3d rope, void *stream) {
  lc_status s = check_common(plan, rope, batch, heads, head_dim, dtype);
  if (s != LC_OK) return s;
  if (!q || !k || !v || !out) return LC_ERR_INVALID_ARGUMENT;
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return LC_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale)) return LC_ERR_INVALID_ARGUMENT;
  // The scheduler counter in the fixed scratch is a 32-bit int: one launch
  // may hand out at most 2^31 - 1 work items (batch x heads x query groups).
  if ((long long)batch * heads * plan->G >= (1LL << 31)) return LC_ERR_UNSUPPORTED;
  float scale = softmax_scale > 0.f ? softmax_scale : 0.125f;
  int *scratch = lc_noalloc_scratch(&s);  // first call on a device: symbol lookup
  if (s != LC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == LC_DTYPE_F32)  // the fp32 kernel needs no scratch
    return lc_launch_forward_f32(static_cast<const float *>(q), static_cast<const float *>(k),
                                 static_cast<const float *>(v), nullptr, nullptr,
                                 static_cast<float *>(out), lse, batch, heads, scale, LC_FWD_FULL,
                                 false, lc_qk_norm(), plan, rope, scratch + 1, st);
  return lc_launch_forward_sm100(q, k, v, nullptr, nullptr, out, lse, batch, heads, scale,
                                 LC_FWD_FULL, false, lc_qk_norm(), plan, rope, scratch + 1, st,
                                 scratch);
}

extern "C" lc_status lc_bsa_forward_shard(const void *q, const void *k, const void *v, void *out,
                                          float *lse, int batch, int heads, int head_dim,
                                          lc_dtype dtype, float softmax_scale,
                                          const lc_bsa_opts *opts, lc_bsa_plan plan,
                                          lc_rope3d rope, void *stream) {
  lc_status s = check_common(plan, rope, batch, heads, head_dim, dtype, true);
  if (s != LC_OK) return s;
  unsigned flags;
  lc_qk_norm norm;
  if (!parse_opts(opts,
                  LC_FLAG_Q_ROTATED | LC_FLAG_K_ROTATED | LC_FLAG_KEEP_EMPTY_ROWS |
                      LC_FLAG_OVERLAP_PREVIOUS,
                  &flags, &norm))
    return LC_ERR_INVALID_ARGUMENT;
  // An overlapping launch must not be preceded by a fill of the rows without keys.
  if ((flags & LC_FLAG_OVERLAP_PREVIOUS) && !(flags & LC_FLAG_KEEP_EMPTY_ROWS))
    return LC_ERR_INVALID_ARGUMENT;
  if (!q || !k || !v || !out || !lse) return LC_ERR_INVALID_ARGUMENT;
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return LC_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale)) return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16) return LC_ERR_UNSUPPORTED;
  const float scale = softmax_scale > 0.f ? softmax_scale : 0.125f;
  lc_shard_view sv;
  sv.q_lo = lc_block_token(plan, plan->qlo);
  sv.q_n = lc_block_token(plan, plan->qhi) - sv.q_lo;
  sv.k_lo = lc_block_token(plan, plan->klo);
  sv.k_n = lc_block_token(plan, plan->khi) - sv.k_lo;
  sv.q_rotated = (flags & LC_FLAG_Q_ROTATED) != 0;
  sv.k_rotated = (flags & LC_FLAG_K_ROTATED) != 0;
  sv.overlap_previous = (flags & LC_FLAG_OVERLAP_PREVIOUS) != 0;
  if (sv.q_n == 0) return LC_OK;
  int *dev_status = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Rows of groups without entries (out = 0, lse = -inf); the kernel writes the rest.
  if (!(flags & LC_FLAG_KEEP_EMPTY_ROWS))
    s = lc_launch_shard_fill(plan, out, lse, batch, heads, dtype, st);
  if (s != LC_OK || plan->G_active == 0) return s;
  return lc_launch_forward_sm100(q, k, v, nullptr, nullptr, out, lse, batch, heads, scale,
                                 LC_FWD_SHARD, false, norm, plan, rope, dev_status, st, nullptr,
                                 &sv);
}

extern "C" lc_status lc_bsa_lse_merge(float *o_acc, float *lse_acc, const void *o_part,
                                      const float *lse_part, void *out, int batch,
                                      long long n_tokens, int heads, int head_dim, lc_dtype dtype,
                                      unsigned flags, void *stream) {
  if (batch <= 0 || heads <= 0 || head_dim <= 0 || n_tokens < 0) return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16 && dtype != LC_DTYPE_F32) return LC_ERR_INVALID_ARGUMENT;
  if (flags & ~(unsigned)LC_MERGE_INIT) return LC_ERR_INVALID_ARGUMENT;
  if (head_dim != LC_HEAD_DIM) return LC_ERR_UNSUPPORTED;
  const bool init = (flags & LC_MERGE_INIT) != 0;
  if (!lse_acc || !o_part || !lse_part || (!o_acc && !(init && out)))
    return LC_ERR_INVALID_ARGUMENT;
  if (misaligned(o_acc) || misaligned(o_part) || misaligned(out) ||
      ((reinterpret_cast<uintptr_t>(lse_acc) | reinterpret_cast<uintptr_t>(lse_part)) & 3u))
    return LC_ERR_INVALID_ARGUMENT;
  if ((long long)batch * n_tokens * heads >= (1LL << 40)) return LC_ERR_UNSUPPORTED;
  return lc_launch_lse_merge(o_acc, lse_acc, o_part, lse_part, out, batch, n_tokens, heads, dtype,
                             init, static_cast<cudaStream_t>(stream));
}

extern "C" lc_status lc_bsa_lse_merge_parts(const void *parts, const float *lses, int n_parts,
                                            void *out, float *lse_out, int batch,
                                            long long n_tokens, int heads, int head_dim,
                                            lc_dtype dtype, void *stream) {
  if (batch <= 0 || heads <= 0 || head_dim <= 0 || n_tokens < 0 || n_parts <= 0)
    return LC_ERR_INVALID_ARGUMENT;
  if (dtype != LC_DTYPE_BF16 && dtype != LC_DTYPE_F32) return LC_ERR_INVALID_ARGUMENT;
  if (head_dim != LC_HEAD_DIM) return LC_ERR_UNSUPPORTED;
  if (!parts || !lses || !out || misaligned(parts) || misaligned(out) ||
      ((reinterpret_cast<uintptr_t>(lses) | reinterpret_cast<uintptr_t>(lse_out)) & 3u))
    return LC_ERR_INVALID_ARGUMENT;
  if ((long long)batch * n_tokens * heads * n_parts >= (1LL << 40)) return LC_ERR_UNSUPPORTED;
  return lc_launch_lse_merge_parts(parts, lses, n_parts, out, lse_out, batch, n_tokens, heads,
                                   dtype, static_cast<cudaStream_t>(stream));
}

extern "C" lc_status lc_last_device_status(void *stream) {
  lc_status s;
  int *p = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  // The allocation-free entry point's status word is read only on a device
  // where that entry point has run (its address was looked up then).
  int *na = lc_noalloc_scratch_if_ready();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LC_CUDA_TRY(cudaStreamSynchronize(st));
  int word = 0, word_na = 0;
  LC_CUDA_TRY(cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost));
  LC_CUDA_TRY(cudaMemset(p, 0, sizeof(int)));
  if (na) {
    LC_CUDA_TRY(cudaMemcpy(&word_na, na + 1, sizeof(int), cudaMemcpyDeviceToHost));
    LC_CUDA_TRY(cudaMemset(na + 1, 0, sizeof(int)));
  }
  return lc_device_status_decode(word | word_na);
}

extern "C" lc_status lc_device_status_decode(int word) {
  if (word & LC_DEVSTAT_TIMEOUT) return LC_ERR_TIMEOUT;
  if (word & LC_DEVSTAT_CHECK) return LC_ERR_DEVICE_CHECK;
  return LC_OK;
}

extern "C" lc_status lc_debug_watchdog_selftest(int timeout_us, void *stream) {
  if (timeout_us <= 0 || timeout_us > 10 * 1000 * 1000) return LC_ERR_INVALID_ARGUMENT;
  lc_status s;
  int *p = lc_device_status_ptr(&s);
  if (s != LC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LC_CUDA_TRY(cudaStreamSynchronize(st));
  LC_CUDA_TRY(cudaMemset(p, 0, sizeof(int)));
  s = lc_launch_watchdog_selftest(p, (long long)timeout_us * 1000LL, st);
  if (s != LC_OK) return s;
  return lc_last_device_status(stream);
}

extern "C" lc_status lc_debug_scratch_pool_used_high(unsigned long long *bytes, int reset) {
  if (!bytes) return LC_ERR_INVALID_ARGUMENT;
  lc_status s;
  cudaMemPool_t pool = lc_scratch_pool(&s);
  if (s != LC_OK) return s;
  if (reset) {
    uint64_t zero = 0;  // resets the mark to the bytes in use now
    LC_CUDA_TRY(cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero));
  }
  uint64_t v = 0;
  LC_CUDA_TRY(cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &v));
  *bytes = (unsigned long long)v;
  return LC_OK;
}

extern "C" const char *lc_status_string(lc_status s) {
  switch (s) {
    case LC_OK: return "ok";
    case LC_ERR_INVALID_ARGUMENT: return "invalid argument";
    case LC_ERR_UNSUPPORTED: return "unsupported configuration";
    case LC_ERR_CUDA: return "CUDA error";
    case LC_ERR_OUT_OF_MEMORY: return "out of device memory";
    case LC_ERR_TIMEOUT: return "a bounded in-kernel wait timed out";
    case LC_ERR_DEVICE_CHECK: return "an in-kernel consistency check failed";
  }
  return "unknown status";
}

extern "C" const char *lc_version(void) { return "0.1.0"; }
