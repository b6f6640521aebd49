// C ABI of the looped GDN mixer library: argument validation, dispatch to the
// kernels, the device status word.  See include/gdn.h for the contract of each
// entry point.
#include <string.h>

#include "common.cuh"

namespace gdn {
bool prefill_tc_supported(const gdn_fwd_params* p);
SegPlan plan_prefill_segments(const gdn_fwd_params* p, int sms);
size_t prefill_segment_workspace(const gdn_fwd_params* p, const SegPlan& plan);
gdn_status launch_prefill_tc(const gdn_fwd_params* p, unsigned* status, const SegPlan& plan, void* ws,
                             cudaStream_t stream);
gdn_status launch_prefill_simt(const gdn_fwd_params* p, unsigned* status, cudaStream_t stream);
gdn_status launch_prefill_kda(const gdn_fwd_params* p, unsigned* status, void* ws, cudaStream_t stream);
size_t prefill_kda_workspace(const gdn_fwd_params* p);
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* a,
                          const float* b, float* S, void* o, const float* gate, const void* h_prev,
                          const float* rho, int N, int H, int dk, int dv, gdn_dtype dt, float scale,
                          unsigned flags, int num_sms, unsigned* status, cudaStream_t stream);
cudaError_t launch_loop_residual(const void* h_tilde, const void* h_prev, const float* rho,
                                 void* h_out, int64_t rows, int d, gdn_dtype dt, int num_sms,
                                 cudaStream_t stream);
gdn_status launch_swa(const swa_params* p, unsigned* status, cudaStream_t stream);
size_t bwd_workspace(const gdn_bwd_params* p);
gdn_status launch_bwd(const gdn_bwd_params* p, unsigned* status, void* ws, cudaStream_t stream);
size_t bwd_chunk_workspace(const gdn_bwd_params* p);
gdn_status launch_bwd_chunk(const gdn_bwd_params* p, unsigned* status, void* ws, cudaStream_t stream);
}  // namespace gdn

// Device status word: kernels record the first error they hit (atomicCAS from 0).
__device__ unsigned g_gdn_device_status = 0;

namespace {

using gdn::kMaxDevices;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Address of the status word on the current device (looked up once per device).
unsigned* status_ptr() {
  static void* cache[kMaxDevices] = {nullptr};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_gdn_device_status) != cudaSuccess) return nullptr;
    cache[dev] = ptr;
  }
  return static_cast<unsigned*>(cache[dev]);
}

int sm_count() {
  static int cache[kMaxDevices] = {0};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool dtype_ok(gdn_dtype t) { return t == GDN_F32 || t == GDN_BF16; }

size_t elem_bytes(gdn_dtype t) { return t == GDN_BF16 ? 2 : 4; }

// A device buffer as a byte range; a null pointer overlaps nothing.
struct Range {
  const void* ptr;
  size_t bytes;
};

template <size_t N>
bool overlaps_any(const Range& x, const Range (&others)[N]) {
  const char* x0 = static_cast<const char*>(x.ptr);
  if (!x0 || x.bytes == 0) return false;
  for (const Range& r : others) {
    const char* r0 = static_cast<const char*>(r.ptr);
    if (r0 && r.bytes && r0 < x0 + x.bytes && x0 < r0 + r.bytes) return true;
  }
  return false;
}

// Shape/pointer checks shared by the workspace query and the launch.
gdn_status validate_fwd(const gdn_fwd_params* p) {
  if (!p) return GDN_ERR_INVALID;
  if (!dtype_ok(p->io_dtype)) return GDN_ERR_INVALID;
  if (p->n_seq < 0 || p->H <= 0 || p->dk <= 0 || p->dv <= 0 || p->total_tokens < 0)
    return GDN_ERR_INVALID;
  if (p->flags & ~(GDN_QK_L2NORM | GDN_PRECISE | GDN_SINGLE_PASS | GDN_CHANNEL_GATE | GDN_TEST_WAIT_TIMEOUT))
    return GDN_ERR_INVALID;
  if (!p->cu_seqlens) {
    if (p->seq_len < 0) return GDN_ERR_INVALID;
    if ((long long)p->n_seq * p->seq_len != (long long)p->total_tokens) return GDN_ERR_INVALID;
  }
  if (p->dk != 64 && p->dk != 128) return GDN_ERR_UNSUPPORTED;
  if (p->dv % 64 != 0 || p->dv > 512) return GDN_ERR_UNSUPPORTED;
  const bool any_tokens = p->total_tokens > 0;
  if (any_tokens && (!p->q || !p->k || !p->v || !p->a || !p->b || !p->o)) return GDN_ERR_INVALID;
  const void* ptrs[] = {p->q, p->k, p->v, p->a, p->b, p->S0, p->o, p->S_T, p->cu_seqlens,
                        p->gate, p->h_prev, p->rho};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return GDN_ERR_INVALID;
  if ((p->h_prev == nullptr) != (p->rho == nullptr)) return GDN_ERR_INVALID;
  if (p->S_T && p->S0 && p->S_T != p->S0) {
    // partial overlap of S0 and S_T is not allowed (exact aliasing is)
    const size_t bytes = (size_t)p->n_seq * p->H * p->dk * p->dv * sizeof(float);
    const char* a0 = reinterpret_cast<const char*>(p->S0);
    const char* b0 = reinterpret_cast<const char*>(p->S_T);
    if (a0 < b0 + bytes && b0 < a0 + bytes) return GDN_ERR_INVALID;
  }
  if (any_tokens && p->o) {
    // the output may not overlap any input or either state
    const size_t tok = (size_t)p->total_tokens * p->H, eb = elem_bytes(p->io_dtype);
    const size_t sb = (size_t)p->n_seq * p->H * p->dk * p->dv * sizeof(float);
    const size_t ab = tok * sizeof(float) * ((p->flags & GDN_CHANNEL_GATE) ? p->dk : 1);
    const Range others[] = {{p->q, tok * p->dk * eb}, {p->k, tok * p->dk * eb},
                            {p->v, tok * p->dv * eb}, {p->a, ab},
                            {p->b, tok * sizeof(float)}, {p->S0, sb}, {p->S_T, sb},
                            {p->gate, tok * sizeof(float)}, {p->rho, (size_t)p->H * p->dv * sizeof(float)},
                            {p->h_prev == p->o ? nullptr : p->h_prev, tok * p->dv * eb}};
    if (overlaps_any({p->o, tok * p->dv * eb}, others)) return GDN_ERR_INVALID;
  }
  return GDN_OK;
}

gdn_status validate_bwd(const gdn_bwd_params* p) {
  if (!p) return GDN_ERR_INVALID;
  if (!dtype_ok(p->io_dtype)) return GDN_ERR_INVALID;
  if (p->n_seq < 0 || p->H <= 0 || p->total_tokens < 0 || p->dk <= 0 || p->dv <= 0) return GDN_ERR_INVALID;
  if ((p->flags & ~GDN_PRECISE) != 0) return GDN_ERR_UNSUPPORTED;
  if (p->dk != 64 && p->dk != 128) return GDN_ERR_UNSUPPORTED;
  if (p->dv % 32 != 0 || p->dv > 256) return GDN_ERR_UNSUPPORTED;
  if (!p->cu_seqlens) {
    if (p->seq_len < 0 || (long long)p->n_seq * p->seq_len != p->total_tokens) return GDN_ERR_INVALID;
  }
  if (p->n_seq == 0) return GDN_OK;
  if (p->total_tokens > 0) {
    const void* need[] = {p->q, p->k, p->v, p->a, p->b, p->grad_o,
                          p->grad_q, p->grad_k, p->grad_v, p->grad_a, p->grad_b};
    for (const void* x : need)
      if (!x || !aligned16(x)) return GDN_ERR_INVALID;
  }
  const void* opt[] = {p->S0, p->grad_S_T, p->grad_S0, p->cu_seqlens};
  for (const void* x : opt)
    if (x && !aligned16(x)) return GDN_ERR_INVALID;
  return GDN_OK;
}

}  // namespace

extern "C" {

size_t gdn_chunk_bwd_workspace(const gdn_bwd_params* p) {
  if (validate_bwd(p) != GDN_OK) return (size_t)-1;
  if (p->n_seq == 0) return 0;
  return (p->flags & GDN_PRECISE) ? gdn::bwd_workspace(p) : gdn::bwd_chunk_workspace(p);
}

gdn_status gdn_chunk_bwd(const gdn_bwd_params* p, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const gdn_status v = validate_bwd(p);
  if (v != GDN_OK) return v;
  if (p->n_seq == 0) return GDN_OK;
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return GDN_ERR_INVALID;
  const bool token = (p->flags & GDN_PRECISE) != 0;
  const size_t need = token ? gdn::bwd_workspace(p) : gdn::bwd_chunk_workspace(p);
  if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
  unsigned* st = status_ptr();
  if (!st) return GDN_ERR_CUDA;
  return token ? gdn::launch_bwd(p, st, ws, stream) : gdn::launch_bwd_chunk(p, st, ws, stream);
}

int gdn_version(void) { return 100; }

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device-side wait timed out";
    case GDN_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

size_t gdn_chunk_fwd_workspace(const gdn_fwd_params* p) {
  if (validate_fwd(p) != GDN_OK) return (size_t)-1;
  if (p->total_tokens == 0 || p->n_seq == 0) return 0;
  if (p->flags & GDN_CHANNEL_GATE) return gdn::prefill_kda_workspace(p);
  return gdn::prefill_segment_workspace(p, gdn::plan_prefill_segments(p, sm_count()));
}

gdn_status gdn_chunk_fwd_schedule(const gdn_fwd_params* p, int* n_segs, int* seg0_tok, int* seg_tok,
                                  int* launches, int* corrected) {
  const gdn_status v = validate_fwd(p);
  if (v != GDN_OK) return v;
  gdn::SegPlan plan{1, 0, 0, 0, 0};
  if (p->total_tokens > 0 && gdn::prefill_tc_supported(p)) plan = gdn::plan_prefill_segments(p, sm_count());
  int n = 1;                                           // one pass
  if (p->n_seq == 0) n = 0;
  else if (p->total_tokens == 0) n = (p->S_T && p->S0 != p->S_T) ? 1 : 0;   // a copy or a clear of S_T
  else if (plan.corrected) n = (plan.n_segs > 2 || p->S_T) ? 3 : 2;          // state pass, combine, correction
  else if (plan.n_segs > 2) n = 3;                                          // state pass, combine, output pass
  else if (plan.n_segs == 2 || plan.lpt) n = 2;
  else if (p->flags & GDN_CHANNEL_GATE) n = 2;                               // the chunks' operands, the chains
  if (n_segs) *n_segs = plan.n_segs;
  if (seg0_tok) *seg0_tok = plan.seg0_tok;
  if (seg_tok) *seg_tok = plan.seg_tok;
  if (launches) *launches = n;
  if (corrected) *corrected = plan.corrected;
  return GDN_OK;
}

gdn_status gdn_chunk_fwd(const gdn_fwd_params* p, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  const gdn_status v = validate_fwd(p);
  if (v != GDN_OK) return v;
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return GDN_ERR_INVALID;
  if (p->n_seq == 0) return GDN_OK;
  if (p->total_tokens == 0) {
    // every sequence is empty: S_T = S0 (or zero)
    if (!p->S_T) return GDN_OK;
    const size_t bytes = (size_t)p->n_seq * p->H * p->dk * p->dv * sizeof(float);
    cudaError_t e = p->S0 ? (p->S0 == p->S_T ? cudaSuccess
                                             : cudaMemcpyAsync(p->S_T, p->S0, bytes,
                                                               cudaMemcpyDeviceToDevice, stream))
                          : cudaMemsetAsync(p->S_T, 0, bytes, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }
  const bool tc = gdn::prefill_tc_supported(p);
  gdn::SegPlan plan = tc ? gdn::plan_prefill_segments(p, sm_count()) : gdn::SegPlan{1, 0, 0, 0, 0};
  if (plan.n_segs > 1 || plan.lpt) {
    const size_t need = gdn::prefill_segment_workspace(p, plan);
    if (!ws && ws_bytes == 0) plan = gdn::SegPlan{1, 0, 0, 0, 0};   // no workspace: one pass, natural order
    else if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
  }
  // per-channel gate: a workspace selects the two launches, none the one-launch kernel
  if ((p->flags & GDN_CHANNEL_GATE) && (ws ? ws_bytes < gdn::prefill_kda_workspace(p) : ws_bytes != 0))
    return GDN_ERR_WORKSPACE;
  unsigned* st = status_ptr();
  if (!st) return GDN_ERR_CUDA;
  if (tc) return gdn::launch_prefill_tc(p, st, plan, ws, stream);
  if (p->flags & GDN_CHANNEL_GATE) return gdn::launch_prefill_kda(p, st, ws, stream);
  return gdn::launch_prefill_simt(p, st, stream);
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, const float* a,
                           const float* b, float* S, void* o, int N, int H, int dk, int dv,
                           gdn_dtype io_dtype, float scale, unsigned flags,
                           cudaStream_t stream) {
  return gdn_decode_step_looped(q, k, v, a, b, S, o, nullptr, nullptr, nullptr, N, H, dk, dv, io_dtype,
                                scale, flags, stream);
}

gdn_status gdn_decode_step_looped(const void* q, const void* k, const void* v, const float* a,
                                  const float* b, float* S, void* o, const float* gate,
                                  const void* h_prev, const float* rho, int N, int H, int dk, int dv,
                                  gdn_dtype io_dtype, float scale, unsigned flags, cudaStream_t stream) {
  if (!dtype_ok(io_dtype) || N < 0 || H <= 0 || dk <= 0 || dv <= 0) return GDN_ERR_INVALID;
  if (flags & ~(GDN_QK_L2NORM | GDN_CHANNEL_GATE)) return GDN_ERR_INVALID;
  if (dk != 64 && dk != 128) return GDN_ERR_UNSUPPORTED;
  if (dv % 64 != 0 || dv > 512) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!q || !k || !v || !a || !b || !S || !o) return GDN_ERR_INVALID;
  if ((h_prev == nullptr) != (rho == nullptr)) return GDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, a, b, S, o};
  for (const void* x : ptrs)
    if (!aligned16(x)) return GDN_ERR_INVALID;
  const void* opt[] = {gate, h_prev, rho};
  for (const void* x : opt)
    if (x && !aligned16(x)) return GDN_ERR_INVALID;
  {
    // o may not overlap the state or any input (other CTAs still read them);
    // h_prev may be o itself (each element is read and then written by one thread)
    const size_t nh = (size_t)N * H, eb = elem_bytes(io_dtype);
    const Range others[] = {{S, nh * dk * dv * sizeof(float)}, {q, nh * dk * eb}, {k, nh * dk * eb},
                            {v, nh * dv * eb},
                            {a, nh * sizeof(float) * ((flags & GDN_CHANNEL_GATE) ? dk : 1)},
                            {b, nh * sizeof(float)}, {gate, nh * sizeof(float)}, {rho, (size_t)H * dv * sizeof(float)},
                            {h_prev == o ? nullptr : h_prev, nh * dv * eb}};
    if (overlaps_any({o, nh * dv * eb}, others)) return GDN_ERR_INVALID;
  }
  const cudaError_t e = gdn::launch_decode(q, k, v, a, b, S, o, gate, h_prev, rho, N, H, dk, dv, io_dtype,
                                           scale, flags, sm_count(), status_ptr(), stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status loop_residual(const void* h_tilde, const void* h_prev, const float* rho, void* h_out,
                         int64_t rows, int d, gdn_dtype io_dtype, cudaStream_t stream) {
  if (!dtype_ok(io_dtype) || rows < 0 || d <= 0 || d % 8 != 0) return GDN_ERR_INVALID;
  if (rows == 0) return GDN_OK;
  if (!h_tilde || !h_prev || !rho || !h_out) return GDN_ERR_INVALID;
  if (!aligned16(h_tilde) || !aligned16(h_prev) || !aligned16(rho) || !aligned16(h_out))
    return GDN_ERR_INVALID;
  const cudaError_t e = gdn::launch_loop_residual(h_tilde, h_prev, rho, h_out, rows, d, io_dtype,
                                                  sm_count(), stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status swa_fwd(const swa_params* p, cudaStream_t stream) {
  if (!p || !dtype_ok(p->io_dtype)) return GDN_ERR_INVALID;
  if (p->n_seq < 0 || p->H <= 0 || p->total_tokens < 0 || p->window < 1 || p->d <= 0 || p->dv <= 0)
    return GDN_ERR_INVALID;
  if (p->io_dtype != GDN_BF16 || p->d != 128 || p->dv != 128) return GDN_ERR_UNSUPPORTED;
  if (p->cu_seqlens) {
    if (p->max_seq_len < 0) return GDN_ERR_INVALID;
  } else if (p->seq_len < 0 || (long long)p->n_seq * p->seq_len != p->total_tokens) {
    return GDN_ERR_INVALID;
  }
  if (p->n_seq == 0 || p->total_tokens == 0) return GDN_OK;
  const void* need[] = {p->q, p->k, p->v, p->o};
  for (const void* x : need)
    if (!x || !aligned16(x)) return GDN_ERR_INVALID;
  if (p->cu_seqlens && !aligned16(p->cu_seqlens)) return GDN_ERR_INVALID;
  const size_t tok = (size_t)p->total_tokens * p->H * 2;
  const Range others[] = {{p->q, tok * p->d}, {p->k, tok * p->d}, {p->v, tok * p->dv}};
  if (overlaps_any({p->o, tok * p->dv}, others)) return GDN_ERR_INVALID;
  unsigned* st = status_ptr();
  if (!st) return GDN_ERR_CUDA;
  return gdn::launch_swa(p, st, stream);
}

gdn_status gdn_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
  unsigned host = 0;
  if (cudaMemcpyFromSymbol(&host, g_gdn_device_status, sizeof(host)) != cudaSuccess)
    return GDN_ERR_CUDA;
  const unsigned zero = 0;
  if (host != 0 && cudaMemcpyToSymbol(g_gdn_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return GDN_ERR_CUDA;
  return static_cast<gdn_status>(host);
}

}  // extern "C"
