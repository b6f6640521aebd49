// Chunkwise prefill of the per-channel (diagonal) gate variant, KDA, with fp32
// operands on the CUDA cores.
//
// KDA is named among the LT2 mixers ("LT2: Linear-Time Looped Transformers",
// Appendix C) and is the DPLR block of §2 / Appendix B.1 with a diagonal
// decay; the pages print no update rule.  The reading used throughout this
// library (state Sigma in R^{dk x dv}, a_t in (0, 1]^{dk}):
//     Sigma_t = (I - b_t k_t k_t^T) Diag(a_t) Sigma_{t-1} + b_t k_t v_t^T,
//     o_t = scale Sigma_t^T q_t.
// Per token, with u_t = b_t (v_t - (Diag(a_t) Sigma_{t-1})^T k_t):
// Sigma_t = Diag(a_t) Sigma_{t-1} + k_t u_t^T.  Unrolled over a chunk of C = 64
// tokens from Sigma_0, with G_ic = sum_{j<=i} log a_jc (every difference
// G_ic - G_jc, j <= i, is <= 0):
//     A_ij  = b_i sum_c k_ic k_jc e^{G_ic - G_jc}      (j < i),  T = (I + A)^{-1}
//     P_ij  = sum_c q_ic k_jc e^{G_ic - G_jc}          (j <= i)
//     U     = T diag(b) (V - (K o e^G) Sigma_0)
//     O     = scale ((Q o e^G) Sigma_0 + P U)
//     Sigma_C = Diag(e^{G_C}) Sigma_0 + (K o e^{G_C - G})^T U
// The decay of each (i, j, c) term is its own exponential (no factorisation
// into e^{G_i} e^{-G_j}, which overflows when a channel decays hard), so every
// exponent is <= 0.  One CTA of 256 threads per (sequence, head, 64-column dv
// slice); the output epilogue (head-wise gate, loop residual) is the precise
// path's.
#include "common.cuh"

namespace gdn {
namespace kda {

constexpr int C = 64;
constexpr int DVS = 64;
constexpr int THREADS = 256;
constexpr int LDC = C + 1;

// T = (I + A)^{-1} for the strictly lower C x C matrix A (row stride LDC in
// shared memory), column `col` per thread: forward substitution with the
// column held in registers, t_i = delta_{i,col} - sum_{m<i} A_im t_m, four
// independent partial sums per row (the entries above the diagonal come out
// zero by themselves: t_m = 0 for m < col).
template <int C, int LDC>
__device__ __forceinline__ void solve_column(const float* sA, float* sT, int col) {
  float t[C];
#pragma unroll
  for (int i = 0; i < C; ++i) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < i; ++m) acc[m & 3] = fmaf(sA[i * LDC + m], t[m], acc[m & 3]);
    t[i] = ((i == col) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
  }
#pragma unroll
  for (int i = 0; i < C; ++i) sT[i * LDC + col] = t[i];
}

template <int DK>
struct Plan {
  static constexpr int LDK = DK + 1;
  static constexpr int K = 0;                      // [C][LDK]  K, then K o e^{G_C - G}
  static constexpr int Q = K + C * LDK;            // [C][LDK]  Q, then Q o e^G
  static constexpr int G = Q + C * LDK;            // [C][LDK]  G, then K o e^G
  static constexpr int SIG = G + C * LDK;          // [DK][LDC] (64 used)
  static constexpr int V = SIG + DK * LDC;         // [C][LDC]  V, then V - (K o e^G) Sigma_0
  static constexpr int A = V + C * LDC;            // [C][LDC]
  static constexpr int T = A + C * LDC;            // [C][LDC]
  static constexpr int P = T + C * LDC;            // [C][LDC]
  static constexpr int U = P + C * LDC;            // [C][LDC]
  static constexpr int B = U + C * LDC;            // b: C
  static constexpr int GC = B + C;                 // e^{G_C}: DK
  static constexpr int FLOATS = GC + DK + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};
static_assert(Plan<128>::BYTES <= 232448, "KDA prefill shared memory");

struct Params {
  const void *q, *k, *v;
  const float *a, *b, *S0;   // a: [tokens][H][dk]
  float* S_T;
  void* o;
  const int32_t* cu_seqlens;
  unsigned* status;
  const float* gate;
  const void* h_prev;
  const float* rho;
  int n_seq, seq_len, total_tokens, H, dv, n_slices;
  float scale;
  unsigned flags;
};

template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_prefill_kda_kernel(const Params p) {
  using PL = Plan<DK>;
  constexpr int LDK = PL::LDK;
  extern __shared__ float sm[];
  float* sK = sm + PL::K;
  float* sQ = sm + PL::Q;
  float* sG = sm + PL::G;
  float* sSig = sm + PL::SIG;
  float* sV = sm + PL::V;
  float* sA = sm + PL::A;
  float* sT = sm + PL::T;
  float* sP = sm + PL::P;
  float* sU = sm + PL::U;
  float* sb = sm + PL::B;
  float* sgc = sm + PL::GC;

  const int tid = threadIdx.x;
  const int slice = blockIdx.x % p.n_slices;
  const int chain = blockIdx.x / p.n_slices;
  const int h = chain % p.H;
  const int seq = chain / p.H;
  const int H = p.H, dv = p.dv;
  int seq_start, seq_end;
  if (p.cu_seqlens) {
    seq_start = p.cu_seqlens[seq];
    seq_end = p.cu_seqlens[seq + 1];
  } else {
    seq_start = seq * p.seq_len;
    seq_end = seq_start + p.seq_len;
  }
  {
    const int s0 = min(max(seq_start, 0), p.total_tokens);
    const int s1 = min(max(seq_end, s0), p.total_tokens);
    if ((s0 != seq_start || s1 != seq_end) && tid == 0) record_status(p.status, GDN_ERR_INVALID);
    seq_start = s0;
    seq_end = s1;
  }
  const int col0 = slice * DVS;
  const size_t sbase = ((size_t)seq * H + h) * DK * (size_t)dv + col0;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  T* o = static_cast<T*>(p.o);

  for (int e = tid; e < DK * DVS; e += THREADS) {
    const int d = e / DVS, c = e % DVS;
    sSig[d * LDC + c] = p.S0 ? p.S0[sbase + (size_t)d * dv + c] : 0.f;
  }

  for (int tok0 = seq_start; tok0 < seq_end; tok0 += C) {
    const int valid = min(C, seq_end - tok0);
    __syncthreads();
    // ---- load the chunk; rows past the sequence end: zero keys, queries and
    // values, log a = 0, b = 0
    for (int e = tid; e < C * DK; e += THREADS) {
      const int i = e / DK, d = e % DK;
      float kv = 0.f, qv = 0.f, la = 0.f;
      if (i < valid) {
        const size_t off = ((size_t)(tok0 + i) * H + h) * DK + d;
        kv = to_f32(k[off]);
        qv = to_f32(q[off]);
        la = logf(p.a[off]);
      }
      sK[i * LDK + d] = kv;
      sQ[i * LDK + d] = qv;
      sG[i * LDK + d] = la;
    }
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      sV[i * LDC + c] = (i < valid) ? to_f32(v[((size_t)(tok0 + i) * H + h) * dv + col0 + c]) : 0.f;
    }
    if (tid < C) sb[tid] = (tid < valid) ? p.b[(size_t)(tok0 + tid) * H + h] : 0.f;
    __syncthreads();
    // ---- G = prefix sums of log a down each channel (one thread per channel);
    // the q/k L2 norm (threads 128 .. 255, one row each), rounded to the io dtype
    if (tid < DK) {
      float acc = 0.f;
      for (int i = 0; i < C; ++i) {
        acc += sG[i * LDK + tid];
        sG[i * LDK + tid] = acc;
      }
    }
    if ((p.flags & GDN_QK_L2NORM) && tid >= 128 && tid < 128 + 2 * C) {
      const int r = tid - 128;
      float* row = (r < C) ? sK + r * LDK : sQ + (r - C) * LDK;
      float ss = 0.f;
      for (int d = 0; d < DK; ++d) ss = fmaf(row[d], row[d], ss);
      const float inv = 1.0f / sqrtf(ss + kQkNormEps);
      for (int d = 0; d < DK; ++d) row[d] = to_f32(from_f32<T>(row[d] * inv));
    }
    __syncthreads();
    // ---- A and P, each term with its own decay e^{G_ic - G_jc} (the fast
    // exponential: a few ulp on arguments <= 0, far inside the fp32 bar)
    // (only the lower triangle j <= i is enumerated; the upper one is zero)
    for (int e = tid; e < C * (C + 1) / 2; e += THREADS) {
      int i = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
      while (i * (i + 1) / 2 > e) --i;
      while ((i + 1) * (i + 2) / 2 <= e) ++i;
      const int j = e - i * (i + 1) / 2;
      float kk = 0.f, qk = 0.f;
#pragma unroll 8
      for (int d = 0; d < DK; ++d) {
        const float dec = __expf(sG[i * LDK + d] - sG[j * LDK + d]);
        const float kj = sK[j * LDK + d] * dec;
        kk = fmaf(sK[i * LDK + d], kj, kk);
        qk = fmaf(sQ[i * LDK + d], kj, qk);
      }
      sA[i * LDC + j] = (j < i) ? sb[i] * kk : 0.f;
      sP[i * LDC + j] = qk;
    }
    for (int e = tid; e < C * (C - 1) / 2; e += THREADS) {   // the strict upper triangle
      int j = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
      while (j * (j + 1) / 2 > e) --j;
      while ((j + 1) * (j + 2) / 2 <= e) ++j;
      const int i = e - j * (j + 1) / 2;            // i <= j, then shifted: column j + 1 > row i
      sA[i * LDC + j + 1] = 0.f;
      sP[i * LDC + j + 1] = 0.f;
    }
    if (tid < DK) sgc[tid] = sG[(C - 1) * LDK + tid];   // G_C (rows past the end keep it)
    __syncthreads();
    // ---- T = (I + A)^{-1}, one column per thread; meanwhile the decayed
    // operands: Q o e^G over Q, K o e^G over G, K o e^{G_C - G} over K
    if (tid < C) {
      solve_column<C, LDC>(sA, sT, tid);
    } else {
      for (int e = tid - C; e < C * DK; e += THREADS - C) {
        const int i = e / DK, d = e % DK;
        const float g = sG[i * LDK + d];
        const float eg = expf(g);
        const float kv = sK[i * LDK + d];
        sQ[i * LDK + d] *= eg;
        sG[i * LDK + d] = kv * eg;
        sK[i * LDK + d] = kv * expf(sgc[d] - g);
      }
    }
    __syncthreads();
    if (tid < DK) sgc[tid] = expf(sgc[tid]);          // e^{G_C}, for the carry
    // ---- X = V - (K o e^G) Sigma_0, in place of V
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      float acc = sV[i * LDC + c];
      for (int d = 0; d < DK; ++d) acc = fmaf(-sG[i * LDK + d], sSig[d * LDC + c], acc);
      sV[i * LDC + c] = acc;
    }
    __syncthreads();
    // ---- U = T diag(b) X
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc = fmaf(sT[i * LDC + j] * sb[j], sV[j * LDC + c], acc);
      sU[i * LDC + c] = acc;
    }
    __syncthreads();
    // ---- O = scale ((Q o e^G) Sigma_0 + P U), then the output gate and the
    // loop residual (as the precise path)
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      if (i >= valid) continue;
      float qs = 0.f, pu = 0.f;
      for (int d = 0; d < DK; ++d) qs = fmaf(sQ[i * LDK + d], sSig[d * LDC + c], qs);
      for (int j = 0; j <= i; ++j) pu = fmaf(sP[i * LDC + j], sU[j * LDC + c], pu);
      float y = p.scale * (qs + pu);
      const size_t off = ((size_t)(tok0 + i) * H + h) * dv + col0 + c;
      if (p.gate) y *= 1.f / (1.f + __expf(-p.gate[(size_t)(tok0 + i) * H + h]));
      if (p.h_prev) {
        const float hp = to_f32(static_cast<const T*>(p.h_prev)[off]);
        y = fmaf(p.rho[(size_t)h * dv + col0 + c], hp, to_f32(from_f32<T>(y)));
      }
      o[off] = from_f32<T>(y);
    }
    __syncthreads();
    // ---- Sigma_C = Diag(e^{G_C}) Sigma_0 + (K o e^{G_C - G})^T U
    for (int e = tid; e < DK * DVS; e += THREADS) {
      const int d = e / DVS, c = e % DVS;
      float acc = 0.f;
      for (int i = 0; i < C; ++i) acc = fmaf(sK[i * LDK + d], sU[i * LDC + c], acc);
      sSig[d * LDC + c] = fmaf(sgc[d], sSig[d * LDC + c], acc);
    }
  }
  __syncthreads();
  if (p.S_T) {
    for (int e = tid; e < DK * DVS; e += THREADS) {
      const int d = e / DVS, c = e % DVS;
      p.S_T[sbase + (size_t)d * dv + c] = sSig[d * LDC + c];
    }
  }
}

template <int DK, typename T>
static cudaError_t launch_t(const Params& kp, long long blocks, cudaStream_t stream) {
  static std::atomic<bool> attr_set[kMaxDevices];
  const size_t bytes = Plan<DK>::BYTES;
  const cudaError_t e = smem_attr_once(attr_set, gdn_prefill_kda_kernel<DK, T>, bytes);
  if (e != cudaSuccess) return e;
  gdn_prefill_kda_kernel<DK, T><<<(unsigned)blocks, THREADS, bytes, stream>>>(kp);
  return cudaGetLastError();
}

}  // namespace kda

gdn_status launch_prefill_kda(const gdn_fwd_params* p, unsigned* status, cudaStream_t stream) {
  kda::Params kp;
  kp.q = p->q;
  kp.k = p->k;
  kp.v = p->v;
  kp.a = p->a;
  kp.b = p->b;
  kp.S0 = p->S0;
  kp.S_T = p->S_T;
  kp.o = p->o;
  kp.cu_seqlens = p->cu_seqlens;
  kp.status = status;
  kp.gate = p->gate;
  kp.h_prev = p->h_prev;
  kp.rho = p->rho;
  kp.n_seq = p->n_seq;
  kp.seq_len = p->seq_len;
  kp.total_tokens = p->total_tokens;
  kp.H = p->H;
  kp.dv = p->dv;
  kp.n_slices = p->dv / kda::DVS;
  kp.scale = p->scale;
  kp.flags = p->flags;
  const long long blocks = (long long)p->n_seq * p->H * kp.n_slices;
  if (blocks <= 0) return GDN_OK;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  cudaError_t e;
  if (p->io_dtype == GDN_BF16)
    e = p->dk == 128 ? kda::launch_t<128, __nv_bfloat16>(kp, blocks, stream)
                     : kda::launch_t<64, __nv_bfloat16>(kp, blocks, stream);
  else
    e = p->dk == 128 ? kda::launch_t<128, float>(kp, blocks, stream)
                     : kda::launch_t<64, float>(kp, blocks, stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
