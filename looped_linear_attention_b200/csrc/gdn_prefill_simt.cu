// Chunkwise prefill of the gated delta rule with fp32 operands on the CUDA
// cores: the precise path (fp32 inputs, dk = 64, dv slices of 64, or the
// GDN_PRECISE flag).  Same chunked algebra as the tensor-core kernel
// (C = 64 tokens, state Sigma in R^{dk x dv}; "LT2: Linear-Time Looped
// Transformers", §2, "LT2." paragraph, Gated DeltaNet mixer):
//     A = strict_lower(diag(b)(D o K K^T)),  T = (I + A)^{-1},  P = tril(D o Q K^T)
//     W = T diag(b gamma) K,  U = T diag(b) V - W Sigma_0
//     O = scale (diag(gamma) Q Sigma_0 + P U)
//     Sigma_C = gamma_C Sigma_0 + K^T diag(gamma_C/gamma) U
// but with every product in fp32 in shared memory, so the result matches the
// token-by-token recurrence to fp32 rounding.  One CTA of 256 threads owns
// one (sequence, head, 64-column dv slice); the chunk loop is sequential.
#include "common.cuh"

namespace gdn {
namespace simt {

constexpr int C = 64;
constexpr int DVS = 64;
constexpr int THREADS = 256;
constexpr int LDC = C + 1;   // padded row of a C-wide tile

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
  static constexpr int K = 0;                      // [C][LDK]
  static constexpr int Q = K + C * LDK;            // [C][LDK]
  static constexpr int W = Q + C * LDK;            // [C][LDK]
  static constexpr int SIG = W + C * LDK;          // [DK][LDC] (64 used)
  static constexpr int V = SIG + DK * LDC;         // [C][LDC]
  static constexpr int A = V + C * LDC;            // [C][LDC]
  static constexpr int T = A + C * LDC;            // [C][LDC]
  static constexpr int P = T + C * LDC;            // [C][LDC]
  static constexpr int U = P + C * LDC;            // [C][LDC]
  static constexpr int G = U + C * LDC;            // g, gamma, b, gamma_C / gamma: 4 x C
  static constexpr int FLOATS = G + 4 * C + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

struct Params {
  const void *q, *k, *v;
  const float *a, *b, *S0;
  float* S_T;
  void* o;
  const int32_t* cu_seqlens;
  unsigned* status;
  const float* gate;     // [tokens][H] output-gate logits, or null
  const void* h_prev;    // [tokens][H*dv] loop residual input (io dtype), or null
  const float* rho;      // [H*dv]
  int n_seq, seq_len, total_tokens, H, dv, n_slices;
  float scale;
  unsigned flags;
};

template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_prefill_simt_kernel(const Params p) {
  using PL = Plan<DK>;
  constexpr int LDK = PL::LDK;
  extern __shared__ float sm[];
  float* sK = sm + PL::K;
  float* sQ = sm + PL::Q;
  float* sW = sm + PL::W;
  float* sSig = sm + PL::SIG;
  float* sV = sm + PL::V;
  float* sA = sm + PL::A;
  float* sT = sm + PL::T;
  float* sP = sm + PL::P;
  float* sU = sm + PL::U;
  float* sg = sm + PL::G;
  float* sgam = sg + C;
  float* sb = sg + 2 * C;
  float* sr = sg + 3 * C;

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
    // offsets outside [0, total_tokens] or decreasing: clamp, and report
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
    // ---- load the chunk (rows past the sequence end are zero)
    for (int e = tid; e < C * DK; e += THREADS) {
      const int i = e / DK, d = e % DK;
      float kv = 0.f, qv = 0.f;
      if (i < valid) {
        const size_t off = ((size_t)(tok0 + i) * H + h) * DK + d;
        kv = to_f32(k[off]);
        qv = to_f32(q[off]);
      }
      sK[i * LDK + d] = kv;
      sQ[i * LDK + d] = qv;
    }
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      sV[i * LDC + c] = (i < valid) ? to_f32(v[((size_t)(tok0 + i) * H + h) * dv + col0 + c]) : 0.f;
    }
    if (tid < C) {
      float la = 0.f, bb = 0.f;
      if (tid < valid) {
        const size_t ti = (size_t)(tok0 + tid) * H + h;
        la = logf(p.a[ti]);
        bb = p.b[ti];
      }
      sg[tid] = la;
      sb[tid] = bb;
    }
    __syncthreads();
    if (tid == 0) {
      float acc = 0.f;
      for (int i = 0; i < C; ++i) {
        acc += sg[i];
        sg[i] = acc;
      }
    }
    if ((p.flags & GDN_QK_L2NORM) && tid >= 128 && tid < 128 + 2 * C) {
      const int r = tid - 128;
      float* row = (r < C) ? sK + r * LDK : sQ + (r - C) * LDK;
      float ss = 0.f;
      for (int d = 0; d < DK; ++d) ss = fmaf(row[d], row[d], ss);
      const float inv = 1.0f / sqrtf(ss + kQkNormEps);
      for (int d = 0; d < DK; ++d) {
        const float x = row[d] * inv;
        row[d] = to_f32(from_f32<T>(x));   // the normalised vector in the io dtype
      }
    }
    __syncthreads();
    if (tid < C) {
      sgam[tid] = expf(sg[tid]);
      sr[tid] = expf(sg[C - 1] - sg[tid]);   // gamma_C / gamma_i (never 0 / 0)
    }
    // ---- A and P
    for (int e = tid; e < C * C; e += THREADS) {
      const int i = e / C, j = e % C;
      float kk = 0.f, qk = 0.f;
      if (j <= i) {
        for (int d = 0; d < DK; ++d) {
          kk = fmaf(sK[i * LDK + d], sK[j * LDK + d], kk);
          qk = fmaf(sQ[i * LDK + d], sK[j * LDK + d], qk);
        }
      }
      const float dec = (j <= i) ? expf(sg[i] - sg[j]) : 0.f;
      sA[i * LDC + j] = (j < i) ? sb[i] * dec * kk : 0.f;
      sP[i * LDC + j] = dec * qk;
    }
    __syncthreads();
    // ---- T = (I + A)^{-1}, one column per thread
    if (tid < C) {
      solve_column<C, LDC>(sA, sT, tid);
    }
    __syncthreads();
    // ---- W = T diag(b gamma) K,  U~ = T diag(b) V
    for (int e = tid; e < C * DK; e += THREADS) {
      const int i = e / DK, d = e % DK;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc = fmaf(sT[i * LDC + j] * sb[j] * sgam[j], sK[j * LDK + d], acc);
      sW[i * LDK + d] = acc;
    }
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc = fmaf(sT[i * LDC + j] * sb[j], sV[j * LDC + c], acc);
      sU[i * LDC + c] = acc;
    }
    __syncthreads();
    // ---- U = U~ - W Sigma_0
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      float acc = sU[i * LDC + c];
      for (int d = 0; d < DK; ++d) acc = fmaf(-sW[i * LDK + d], sSig[d * LDC + c], acc);
      sU[i * LDC + c] = acc;
    }
    __syncthreads();
    // ---- O = scale (diag(gamma) Q Sigma_0 + P U), then the output gate and
    // the loop residual (o rounded to the io dtype first, as loop_residual sees
    // it; h_prev is read by the thread that then writes the same element)
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      if (i >= valid) continue;
      float qs = 0.f, pu = 0.f;
      for (int d = 0; d < DK; ++d) qs = fmaf(sQ[i * LDK + d], sSig[d * LDC + c], qs);
      for (int j = 0; j <= i; ++j) pu = fmaf(sP[i * LDC + j], sU[j * LDC + c], pu);
      float y = p.scale * fmaf(sgam[i], qs, pu);
      const size_t off = ((size_t)(tok0 + i) * H + h) * dv + col0 + c;
      if (p.gate) y *= 1.f / (1.f + __expf(-p.gate[(size_t)(tok0 + i) * H + h]));
      if (p.h_prev) {
        const float hp = to_f32(static_cast<const T*>(p.h_prev)[off]);
        y = fmaf(p.rho[(size_t)h * dv + col0 + c], hp, to_f32(from_f32<T>(y)));
      }
      o[off] = from_f32<T>(y);
    }
    __syncthreads();
    // ---- Sigma_C = gamma_C Sigma_0 + K^T diag(gamma_C / gamma) U
    const float gC = sgam[C - 1];
    for (int e = tid; e < DK * DVS; e += THREADS) {
      const int d = e / DVS, c = e % DVS;
      float acc = 0.f;
      for (int i = 0; i < C; ++i) acc = fmaf(sK[i * LDK + d] * sr[i], sU[i * LDC + c], acc);
      sSig[d * LDC + c] = fmaf(gC, sSig[d * LDC + c], acc);
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
  const cudaError_t e = smem_attr_once(attr_set, gdn_prefill_simt_kernel<DK, T>, bytes);
  if (e != cudaSuccess) return e;
  gdn_prefill_simt_kernel<DK, T><<<(unsigned)blocks, THREADS, bytes, stream>>>(kp);
  return cudaGetLastError();
}

}  // namespace simt

gdn_status launch_prefill_simt(const gdn_fwd_params* p, unsigned* status, cudaStream_t stream) {
  simt::Params kp;
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
  kp.n_slices = p->dv / simt::DVS;
  kp.scale = p->scale;
  kp.flags = p->flags;
  const long long blocks = (long long)p->n_seq * p->H * kp.n_slices;
  if (blocks <= 0) return GDN_OK;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  cudaError_t e;
  if (p->io_dtype == GDN_BF16)
    e = p->dk == 128 ? simt::launch_t<128, __nv_bfloat16>(kp, blocks, stream)
                     : simt::launch_t<64, __nv_bfloat16>(kp, blocks, stream);
  else
    e = p->dk == 128 ? simt::launch_t<128, float>(kp, blocks, stream)
                     : simt::launch_t<64, float>(kp, blocks, stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
