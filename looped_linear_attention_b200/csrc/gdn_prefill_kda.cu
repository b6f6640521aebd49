// Chunkwise prefill of the per-channel (diagonal) gate variant, KDA, in fp32:
// CUDA-core kernels, the chain launch's two products on warp-level 3xTF32
// MMAs (fp32 accumulate).
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
// When every channel's decay over the chunk is moderate (G_0c - G_{C-1,c} <=
// kFactorRange), the decay factors split around the channel's midpoint m_c,
// e^{G_ic - G_jc} = e^{G_ic - m_c} e^{m_c - G_jc} (each factor within
// e^{+-kFactorRange/2}), and A and P become plain products:
// A = diag(b) K~ K^^T and P = Q~ K^^T (lower parts) with K~ = K o e^{G-m},
// K^ = K o e^{m-G}, Q~ = Q o e^{G-m}: two exponentials per (i, c) instead of
// one per (i, j, c).
// Otherwise (a channel that decays hard or resets) the decay of each (i, j, c)
// term is its own exponential, so every exponent is <= 0.  Without a
// workspace one kernel (one CTA of 256 threads per (sequence, head, 32-column
// dv slice)) does all of it; with one, a chunk-parallel launch and a chain
// launch split it (the two-launch section below).  The output epilogue
// (head-wise gate, loop residual) is the precise path's.
#include "common.cuh"
#include "tma_host.h"

namespace gdn {
namespace kda {

constexpr int C = 64;
constexpr int DVS = 32;           // dv columns per CTA (more CTAs for few chains)
constexpr int THREADS = 256;
constexpr int LDC = C + 4;        // C x C and [rows][DVS] tiles: float4 rows
constexpr float kFactorRange = 80.f;   // largest per-channel log-decay range of a factored chunk

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
// TN consecutive floats from / to shared memory (one float2 or float4 access)
template <int TN>
__device__ __forceinline__ void ldv(const float* p, float (&v)[TN]) {
  if constexpr (TN == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else if constexpr (TN == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = *p;
  }
}
template <int TN>
__device__ __forceinline__ void stv(float* p, const float (&v)[TN]) {
  if constexpr (TN == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  else if constexpr (TN == 2) *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  else *p = v[0];
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}

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

// T = (I + A)^{-1} for the strictly lower C x C matrix A (row stride LDC) by
// 16 x 16 blocks (every thread of the CTA calls it; ends with the block
// synced): the four diagonal blocks by forward substitution, one column per
// thread, then block row by block row T_RC = -T_RR sum_{C <= m < R} A_Rm T_mC,
// the sums staged in sX (3 x 256 floats).  The same T as column-wise forward
// substitution up to rounding order.
__device__ __forceinline__ void solve_blocked(const float* sA, float* sT, float* sX, int tid) {
  static_assert(C == 64, "four 16 x 16 blocks");
  if (tid < C) {
    const int R = tid >> 4, col = tid & 15, o = 16 * R;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < i; ++m) acc[m & 3] = fmaf(sA[(o + i) * LDC + o + m], t[m], acc[m & 3]);
      t[i] = ((i == col) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sT[(o + i) * LDC + o + col] = t[i];
  } else {
    // the blocks above the diagonal are zero
    for (int e = tid - C; e < 6 * 256; e += THREADS - C) {
      const int b = e >> 8, w = e & 255;
      const int R = (b >= 5) ? 2 : (b >= 3) ? 1 : 0;
      const int Cb = (b >= 5) ? 3 : (b >= 3) ? b - 1 : b + 1;
      sT[(16 * R + (w >> 4)) * LDC + 16 * Cb + (w & 15)] = 0.f;
    }
  }
  __syncthreads();
#pragma unroll 1
  for (int R = 1; R < 4; ++R) {
    // X_Rc = sum_{c <= m < R} A_Rm T_mc for the R blocks c < R
    for (int e = tid; e < R * 256; e += THREADS) {
      const int c = e >> 8, i = (e >> 4) & 15, j = e & 15;
      const float* arow = sA + (16 * R + i) * LDC;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int m = c; m < R; ++m) {
        const float* tcol = sT + 16 * m * LDC + 16 * c + j;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc[k & 3] = fmaf(arow[16 * m + k], tcol[k * LDC], acc[k & 3]);
      }
      sX[e] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
    // T_Rc = -T_RR X_Rc (T_RR is lower triangular, its upper part zero)
    for (int e = tid; e < R * 256; e += THREADS) {
      const int c = e >> 8, i = (e >> 4) & 15, j = e & 15;
      const float* trow = sT + (16 * R + i) * LDC + 16 * R;
      const float* xcol = sX + c * 256 + j;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k & 3] = fmaf(trow[k], xcol[16 * k], acc[k & 3]);
      sT[(16 * R + i) * LDC + 16 * c + j] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
    }
    __syncthreads();
  }
}

template <int DK>
struct Plan {
  static constexpr int LDK = DK + 4;               // float4 rows (the factored A and P products)
  static constexpr int K = 0;                      // [C][LDK]  K, then K o e^{G_C - G}
  static constexpr int Q = K + C * LDK;            // [C][LDK]  Q, then Q o e^G
  static constexpr int G = Q + C * LDK;            // [C][LDK]  G, then K o e^G
  static constexpr int SIG = G + C * LDK;          // [DK][LDC] (DVS columns used)
  static constexpr int V = SIG + DK * LDC;         // [C][LDC]  V, then V - (K o e^G) Sigma_0
  static constexpr int A = V + C * LDC;            // [C][LDC]
  static constexpr int T = A + C * LDC;            // [C][LDC]
  static constexpr int P = T + C * LDC;            // [C][LDC]
  static constexpr int U = P + C * LDC;            // [C][LDC]
  static constexpr int B = U + C * LDC;            // b: C
  static constexpr int GC = B + C;                 // e^{G_C}: DK
  static constexpr int MID = GC + DK;              // factored chunks: m, e^m, e^{G_C - m}: 3 x DK
  static constexpr int FLOATS = MID + 3 * DK + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};
static_assert(Plan<128>::BYTES <= 232448, "KDA prefill shared memory");

// Workspace of the two-launch schedule, per (chunk slot, head): the chunk's
// operands once the state-independent products are folded in (W, Q', U~ and
// O~ below) and its decay over the chunk.
struct Ws {
  float *W, *Qp;         // [slots][H][C][dk]: T diag(b) (K o e^G), Q o e^G - P W
  float* KhT;            // [slots][H][dk][C]: (K o e^{G_C - G})^T
  float *Ut, *Ot;        // [slots][H][C][dv]: U~ = T diag(b) V, O~ = P U~
  float* EGC;            // [slots][H][dk]: e^{G_C}
  long long n_slots;
};

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
  Ws ws;
};

// A = diag(b) K~ K^^T (strictly lower) and P = Q~ K^^T (lower) of a factored
// chunk, with K^ in the plan's K rows, K~ in its G rows, Q~ in its Q rows.
// Only the ten 16 x 16 macro tiles on or below the diagonal are multiplied:
// 16 threads each, a thread taking rows 16 R + a + 4 i and columns
// 16 Cc + c + 4 j (i, j < 4), so that the eight lanes of a quarter warp read
// two rows of one operand and four of the other, all in distinct banks
// (row stride LDK = 4 mod 32 floats); the other 96 threads zero the six
// macro tiles above the diagonal.
template <int DK, typename PL>
__device__ __forceinline__ void ap_factored(float* sm, int tid) {
  constexpr int LDK = PL::LDK;
  const float* sK = sm + PL::K;
  const float* sQ = sm + PL::Q;
  const float* sG = sm + PL::G;
  const float* sb = sm + PL::B;
  float* sA = sm + PL::A;
  float* sP = sm + PL::P;
  if (tid < 160) {
    const int t = tid >> 4;                        // macro tile, row-band order
    const int R = (t >= 6) ? 3 : (t >= 3) ? 2 : (t >= 1) ? 1 : 0;
    const int Cc = t - R * (R + 1) / 2;
    const int ra = 16 * R + ((tid >> 2) & 3), cb = 16 * Cc + (tid & 3);
    float kk[4][4], qk[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) kk[i][j] = qk[i][j] = 0.f;
#pragma unroll 2
    for (int d = 0; d < DK; d += 4) {
      float4 ak[4], aq[4], bk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ak[i] = lds4(sG + (ra + 4 * i) * LDK + d);
        aq[i] = lds4(sQ + (ra + 4 * i) * LDK + d);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) bk[j] = lds4(sK + (cb + 4 * j) * LDK + d);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          kk[i][j] = dot4(ak[i], bk[j], kk[i][j]);
          qk[i][j] = dot4(aq[i], bk[j], qk[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = ra + 4 * i, cc = cb + 4 * j;
        sA[r * LDC + cc] = (cc < r) ? sb[r] * kk[i][j] : 0.f;
        sP[r * LDC + cc] = (cc <= r) ? qk[i][j] : 0.f;
      }
  } else {
    // macro tiles above the diagonal: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
    for (int e = tid - 160; e < 6 * 256; e += THREADS - 160) {
      const int t = e >> 8, w = e & 255;
      const int R = (t >= 5) ? 2 : (t >= 3) ? 1 : 0;
      const int Cc = (t >= 5) ? 3 : (t >= 3) ? t - 1 : t + 1;
      const int r = 16 * R + (w >> 4), cc = 16 * Cc + (w & 15);
      sA[r * LDC + cc] = 0.f;
      sP[r * LDC + cc] = 0.f;
    }
  }
}

// A and P with each term's own decay e^{G_ic - G_jc} (the fast exponential: a
// few ulp on arguments <= 0, far inside the fp32 bar), from K, Q and G in the
// plan's rows; only the lower triangle j <= i is enumerated, the upper one is
// written as zeros.
template <int DK, typename PL>
__device__ __forceinline__ void ap_exact(float* sm, int tid) {
  constexpr int LDK = PL::LDK;
  const float* sK = sm + PL::K;
  const float* sQ = sm + PL::Q;
  const float* sG = sm + PL::G;
  const float* sb = sm + PL::B;
  float* sA = sm + PL::A;
  float* sP = sm + PL::P;
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
}

// The chunk's operands of the KDA form (every thread of the CTA calls it):
// K, Q (with the q/k norm rounded to the io dtype) and the per-channel log
// decay prefix G of the chunk starting at tok0 (valid rows, zeros below), b,
// A and P (factored when the chunk's decay range allows), T = (I + A)^{-1},
// and the decayed operands written over K, Q and G: K o e^{G_C - G} over K,
// Q o e^G over Q, K o e^G over G; sgc = e^{G_C}.  Ends with the block synced.
template <int DK, typename T, typename PL>
__device__ __forceinline__ void kda_chunk_operands(const Params& p, int tok0, int valid, int h, float* sm, int tid) {
  constexpr int LDK = PL::LDK;
  float* sK = sm + PL::K;
  float* sQ = sm + PL::Q;
  float* sG = sm + PL::G;
  float* sA = sm + PL::A;
  float* sT = sm + PL::T;
  float* sP = sm + PL::P;
  float* sb = sm + PL::B;
  float* sgc = sm + PL::GC;
  float* smid = sm + PL::MID;
  float* sem = smid + DK;
  float* sec = sem + DK;
  const int H = p.H;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
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
  // ---- G_C, the channel midpoints, and whether the chunk factors
  if (tid < DK) {
    const float g0 = sG[tid], gc = sG[(C - 1) * LDK + tid];
    sgc[tid] = gc;                                  // G_C (rows past the end keep it)
    smid[tid] = 0.5f * (g0 + gc);
  }
  const bool factored =
      !__syncthreads_or(tid < DK && !(sG[tid] - sG[(C - 1) * LDK + tid] <= kFactorRange));
  if (factored) {
    // K^ = K o e^{m - G} over K, K~ = K o e^{G - m} over G, Q~ = Q o e^{G - m} over Q
    for (int e = tid; e < C * DK; e += THREADS) {
      const int i = e / DK, d = e % DK;
      const float g = sG[i * LDK + d] - smid[d];
      const float ex = expf(g), fx = expf(-g);
      const float kv = sK[i * LDK + d];
      sK[i * LDK + d] = kv * fx;
      sG[i * LDK + d] = kv * ex;
      sQ[i * LDK + d] *= ex;
    }
    if (tid < DK) {
      sem[tid] = expf(smid[tid]);
      sec[tid] = expf(sgc[tid] - smid[tid]);
    }
    __syncthreads();
    ap_factored<DK, PL>(sm, tid);
    __syncthreads();
    // ---- T = (I + A)^{-1}, one column per thread; meanwhile the decayed
    // operands from the factored ones: Q o e^G = Q~ e^m, K o e^G = K~ e^m,
    // K o e^{G_C - G} = K^ e^{G_C - m}
    if (tid < C) {
      solve_column<C, LDC>(sA, sT, tid);
    } else {
      for (int e = tid - C; e < C * DK; e += THREADS - C) {
        const int i = e / DK, d = e % DK;
        sQ[i * LDK + d] *= sem[d];
        sG[i * LDK + d] *= sem[d];
        sK[i * LDK + d] *= sec[d];
      }
    }
  } else {
    ap_exact<DK, PL>(sm, tid);
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
  }
  __syncthreads();
  if (tid < DK) sgc[tid] = expf(sgc[tid]);          // e^{G_C}, for the carry
  __syncthreads();
}

template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_prefill_kda_kernel(const Params p) {
  using PL = Plan<DK>;
  constexpr int LDK = PL::LDK;
  extern __shared__ __align__(16) float sm[];
  float* sK = sm + PL::K;
  float* sQ = sm + PL::Q;
  float* sG = sm + PL::G;
  float* sSig = sm + PL::SIG;
  float* sV = sm + PL::V;
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
  const T* v = static_cast<const T*>(p.v);
  T* o = static_cast<T*>(p.o);

  for (int e = tid; e < DK * DVS; e += THREADS) {
    const int d = e / DVS, c = e % DVS;
    sSig[d * LDC + c] = p.S0 ? p.S0[sbase + (size_t)d * dv + c] : 0.f;
  }

  for (int tok0 = seq_start; tok0 < seq_end; tok0 += C) {
    const int valid = min(C, seq_end - tok0);
    __syncthreads();
    for (int e = tid; e < C * DVS; e += THREADS) {
      const int i = e / DVS, c = e % DVS;
      sV[i * LDC + c] = (i < valid) ? to_f32(v[((size_t)(tok0 + i) * H + h) * dv + col0 + c]) : 0.f;
    }
    kda_chunk_operands<DK, T, PL>(p, tok0, valid, h, sm, tid);
    // Register tiles from here on: [C][DVS] results give thread rows
    // 4 rg .. 4 rg + 3 and columns TN cg .. TN cg + TN - 1 (rg = tid / 16,
    // cg = tid % 16, TN = DVS / 16); the dk x DVS carry gives it rows DK/16 rg ..
    // and the same columns.
    constexpr int TN = DVS / 16;
    const int rg = tid >> 4, r0 = 4 * rg, c0 = TN * (tid & 15);
    // ---- X = V - (K o e^G) Sigma_0, in place of V
    {
      float acc[4][TN];
#pragma unroll
      for (int i = 0; i < 4; ++i) ldv<TN>(sV + (r0 + i) * LDC + c0, acc[i]);
#pragma unroll 4
      for (int d = 0; d < DK; ++d) {
        float b[TN];
        ldv<TN>(sSig + d * LDC + c0, b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = sG[(r0 + i) * LDK + d];
#pragma unroll
          for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(-a, b[j], acc[i][j]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) stv<TN>(sV + (r0 + i) * LDC + c0, acc[i]);
    }
    __syncthreads();
    // ---- U = T diag(b) X (T is lower triangular: j <= r0 + 3)
    {
      float acc[4][TN] = {};
#pragma unroll 4
      for (int j = 0; j < r0 + 4; ++j) {
        float x[TN];
        ldv<TN>(sV + j * LDC + c0, x);
        const float bj = sb[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = sT[(r0 + i) * LDC + j] * bj;
#pragma unroll
          for (int jj = 0; jj < TN; ++jj) acc[i][jj] = fmaf(a, x[jj], acc[i][jj]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) stv<TN>(sU + (r0 + i) * LDC + c0, acc[i]);
    }
    __syncthreads();
    // ---- O = scale ((Q o e^G) Sigma_0 + P U), then the output gate and the
    // loop residual (as the precise path)
    {
      float acc[4][TN] = {};
#pragma unroll 4
      for (int d = 0; d < DK; ++d) {
        float b[TN];
        ldv<TN>(sSig + d * LDC + c0, b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = sQ[(r0 + i) * LDK + d];
#pragma unroll
          for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a, b[j], acc[i][j]);
        }
      }
#pragma unroll 4
      for (int j = 0; j < r0 + 4; ++j) {
        float u[TN];
        ldv<TN>(sU + j * LDC + c0, u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = sP[(r0 + i) * LDC + j];
#pragma unroll
          for (int jj = 0; jj < TN; ++jj) acc[i][jj] = fmaf(a, u[jj], acc[i][jj]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
        if (r >= valid) continue;
        const float og = p.gate ? 1.f / (1.f + __expf(-p.gate[(size_t)(tok0 + r) * H + h])) : 1.f;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          const int c = c0 + j;
          float y = p.scale * acc[i][j];
          const size_t off = ((size_t)(tok0 + r) * H + h) * dv + col0 + c;
          if (p.gate) y *= og;
          if (p.h_prev) {
            const float hp = to_f32(static_cast<const T*>(p.h_prev)[off]);
            y = fmaf(p.rho[(size_t)h * dv + col0 + c], hp, to_f32(from_f32<T>(y)));
          }
          o[off] = from_f32<T>(y);
        }
      }
    }
    __syncthreads();
    // ---- Sigma_C = Diag(e^{G_C}) Sigma_0 + (K o e^{G_C - G})^T U
    {
      constexpr int TD = DK / 16;
      const int d0 = TD * rg;
      float acc[TD][TN] = {};
#pragma unroll 2
      for (int i = 0; i < C; ++i) {
        float u[TN];
        ldv<TN>(sU + i * LDC + c0, u);
#pragma unroll
        for (int q4 = 0; q4 < TD / 4; ++q4) {
          const float4 a4 = lds4(sK + i * LDK + d0 + 4 * q4);
          const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[4 * q4 + e][j] = fmaf(a[e], u[j], acc[4 * q4 + e][j]);
        }
      }
#pragma unroll
      for (int e = 0; e < TD; ++e) {
        const int d = d0 + e;
        float sg[TN];
        ldv<TN>(sSig + d * LDC + c0, sg);
        const float g = sgc[d];
#pragma unroll
        for (int j = 0; j < TN; ++j) sg[j] = fmaf(g, sg[j], acc[e][j]);
        stv<TN>(sSig + d * LDC + c0, sg);
      }
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

// ---------------------------------------------------------------- two launches
// With a workspace the chunk-parallel part of the form runs once per (chunk,
// head) in a launch of its own: the decayed operands, A, P, T and the
// state-independent products
//     W = T diag(b) (K o e^G),  U~ = T diag(b) V,
//     Q' = Q o e^G - P W,       O~ = P U~,
// and the chains then walk their chunks with only the state-dependent ones:
//     U = U~ - W Sigma_0,  O = scale (Q' Sigma_0 + O~),
//     Sigma_C = Diag(e^{G_C}) Sigma_0 + (K o e^{G_C - G})^T U
// (the same U and O as T diag(b) (V - (K o e^G) Sigma_0) and
// scale ((Q o e^G) Sigma_0 + P U)).
// Chunk c of sequence s (first token t0_s) has workspace slot
// floor(t0_s / C) + s + c: no two chunks share one, and every slot is below
// floor(total / C) + n_seq.

template <int DK>
struct PrepPlan {
  static constexpr int LDK = DK + 4;
  static constexpr int K = 0;                      // [C][LDK]
  static constexpr int Q = K + C * LDK;            // [C][LDK]
  static constexpr int G = Q + C * LDK;            // [C][LDK]
  static constexpr int A = G + C * LDK;            // [C][LDC]
  static constexpr int T = A + C * LDC;            // [C][LDC]
  static constexpr int P = T + C * LDC;            // [C][LDC]
  static constexpr int B = P + C * LDC;            // C
  static constexpr int GC = B + C;                 // DK
  static constexpr int MID = GC + DK;              // 3 x DK
  static constexpr int SX = MID + 3 * DK + 4;      // 3 x 256: the blocked solve's sums
  static constexpr int VST = SX + 3 * 256;         // 2 x [C][64] V rows as loaded (io dtype)
  static constexpr int FLOATS = VST + 2 * C * 64;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};
static_assert(PrepPlan<128>::BYTES <= 232448, "KDA prep shared memory");

__device__ __forceinline__ void seq_range(const Params& p, int s, int& t0, int& t1, bool report) {
  if (p.cu_seqlens) {
    t0 = __ldg(p.cu_seqlens + s);
    t1 = __ldg(p.cu_seqlens + s + 1);
  } else {
    t0 = s * p.seq_len;
    t1 = t0 + p.seq_len;
  }
  const int c0 = min(max(t0, 0), p.total_tokens);
  const int c1 = min(max(t1, c0), p.total_tokens);
  if (report && (c0 != t0 || c1 != t1)) record_status(p.status, GDN_ERR_INVALID);
  t0 = c0;
  t1 = c1;
}
__device__ __forceinline__ long long slot_base(int s, int t0) { return t0 / C + (long long)s; }

// Slot -> (sequence, chunk, first token, rows): the last sequence whose first
// slot is <= slot; false when the slot holds no chunk.
__device__ bool slot_chunk(const Params& p, long long slot, int& tok0, int& valid) {
  int lo = 0, hi = p.n_seq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    int a0, a1;
    seq_range(p, mid, a0, a1, false);
    if (slot_base(mid, a0) <= slot) lo = mid;
    else hi = mid - 1;
  }
  int s0, s1;
  seq_range(p, lo, s0, s1, false);
  const long long c = slot - slot_base(lo, s0);
  if (c < 0 || c >= (s1 - s0 + C - 1) / C) return false;
  tok0 = s0 + (int)c * C;
  valid = min(C, s1 - tok0);
  return true;
}

__device__ __forceinline__ void cp_async16(float* smem, const float* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
// 16 bytes, or zeros when !take (nothing is read then)
__device__ __forceinline__ void cp_async16_or_zero(float* smem, const void* gmem, bool take) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(take ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// rows x W contiguous floats into shared rows of stride LD
template <int ROWS, int W, int LD>
__device__ __forceinline__ void copy_rows(float* dst, const float* src, int tid) {
  for (int e = tid; e < ROWS * W / 4; e += THREADS) {
    const int i = e / (W / 4), c = 4 * (e % (W / 4));
    cp_async16(dst + i * LD + c, src + (size_t)i * W + c);
  }
}

// Four consecutive bf16 values (8 bytes of shared memory) as floats.
__device__ __forceinline__ void lds_bf16x4(const float* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}
__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

// acc[i][4 q + x] = sum over k < kend (a multiple of 4) of A[i][k] B[k][64 q + 4 cg + x]
// for the four rows of A (stride LDC, read four k at a time) and NQ float4
// column groups of B (rows of stride ldb).
template <int NQ>
__device__ __forceinline__ void tri_times(float (&acc)[4][4 * NQ], const float* A, const float* B, int ldb, int cg,
                                          int kend) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4 * NQ; ++c) acc[i][c] = 0.f;
#pragma unroll 2
  for (int k = 0; k < kend; k += 4) {
    float4 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = lds4(A + i * LDC + k);
    float4 b[4][NQ];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int q = 0; q < NQ; ++q) b[kk][q] = lds4(B + (k + kk) * ldb + 64 * q + 4 * cg);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        float* o = acc[i] + 4 * q;
        o[0] = fmaf(a[i].w, b[3][q].x, fmaf(a[i].z, b[2][q].x, fmaf(a[i].y, b[1][q].x, fmaf(a[i].x, b[0][q].x, o[0]))));
        o[1] = fmaf(a[i].w, b[3][q].y, fmaf(a[i].z, b[2][q].y, fmaf(a[i].y, b[1][q].y, fmaf(a[i].x, b[0][q].y, o[1]))));
        o[2] = fmaf(a[i].w, b[3][q].z, fmaf(a[i].z, b[2][q].z, fmaf(a[i].y, b[1][q].z, fmaf(a[i].x, b[0][q].z, o[2]))));
        o[3] = fmaf(a[i].w, b[3][q].w, fmaf(a[i].z, b[2][q].w, fmaf(a[i].y, b[1][q].w, fmaf(a[i].x, b[0][q].w, o[3]))));
      }
  }
}

// One CTA per (chunk slot, head): the chunk's operands into the workspace.
// Each thread holds four channels (4 dq .. 4 dq + 3) of RPT consecutive rows
// in registers (read from the staged rows): the decay prefix runs
// down the thread's rows and then adds the totals of the row groups above,
// the q/k norm is a reduction across the threads of one row group (lanes of
// one warp), and the decayed operands go from registers to the workspace.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_prefill_kda_prep_kernel(const Params p) {
  using PL = PrepPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int QPR = DK / 4;                      // channel quads per row
  constexpr int RG = THREADS / QPR;                // row groups
  constexpr int RPT = C / RG;                      // rows per thread
  static_assert(QPR <= 32 && 32 % QPR == 0 && RG * RPT == C, "prep register map");
  extern __shared__ __align__(16) float sm[];
  float* sK = sm + PL::K;
  float* sQ = sm + PL::Q;
  float* sG = sm + PL::G;
  float* sT = sm + PL::T;
  float* sb = sm + PL::B;
  float* sTot = sm + PL::A;                        // [RG][DK] row-group sums of log a (A comes later)
  float* sRow0 = sm + PL::GC;                      // [DK] log a of row 0
  const int tid = threadIdx.x;
  const long long slot = blockIdx.x / p.H;
  const int h = blockIdx.x % p.H;
  int tok0, valid;
  if (!slot_chunk(p, slot, tok0, valid)) return;
  const int H = p.H;
  const int d0 = 4 * (tid % QPR), rg = tid / QPR, i0 = RPT * rg;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  // ---- the chunk's q and k rows (io dtype; fp32 ones straight into the Q and
  // K rows, bf16 ones into the T and P areas, which are free until the
  // products) and a rows (into G) staged with cp.async, every piece in
  // flight at once; rows past the sequence end read nothing (zero fill)
  constexpr bool kF32 = sizeof(T) == 4;
  constexpr int RAW_LD = kF32 ? LDK : DK / 2;      // floats per staged q / k row
  // 64 columns of the chunk's V rows (io dtype) into staging buffer `buf`
  const T* v = static_cast<const T*>(p.v);
  constexpr int VROW = 64 * (int)sizeof(T) / 4;    // floats per staged V row
  auto stage_v = [&](int vb, int buf) {
    constexpr int VP = 64 * (int)sizeof(T) / 16;   // 16-byte pieces per row
    for (int e = tid; e < C * VP; e += THREADS) {
      const int i = e / VP, c = e % VP;
      const T* src = v + ((size_t)(tok0 + min(i, valid - 1)) * H + h) * p.dv + vb;
      cp_async16_or_zero(sm + PL::VST + buf * C * 64 + i * VROW + 4 * c, reinterpret_cast<const char*>(src) + 16 * c,
                         i < valid);
    }
  };
  float* rq = kF32 ? sQ : sm + PL::T;
  float* rk = kF32 ? sK : sm + PL::P;
  {
    constexpr int QP = DK * (int)sizeof(T) / 16;   // 16-byte pieces per q / k row
    for (int e = tid; e < C * QP; e += THREADS) {
      const int i = e / QP, c = e % QP;
      const size_t off = ((size_t)(tok0 + min(i, valid - 1)) * H + h) * DK;
      cp_async16_or_zero(rq + i * RAW_LD + 4 * c, reinterpret_cast<const char*>(q + off) + 16 * c, i < valid);
      cp_async16_or_zero(rk + i * RAW_LD + 4 * c, reinterpret_cast<const char*>(k + off) + 16 * c, i < valid);
    }
    for (int e = tid; e < C * DK / 4; e += THREADS) {
      const int i = e / (DK / 4), c = 4 * (e % (DK / 4));
      const size_t off = ((size_t)(tok0 + min(i, valid - 1)) * H + h) * DK;
      cp_async16_or_zero(sG + i * LDK + c, p.a + off + c, i < valid);
    }
    stage_v(0, 0);
    cp_async_commit();
  }
  if (tid < C) sb[tid] = (tid < valid) ? p.b[(size_t)(tok0 + tid) * H + h] : 0.f;
  cp_async_wait<0>();
  __syncthreads();
  // ---- this thread's rows into registers (rows past the end: zero keys and
  // queries, a = 1)
  float kr[RPT][4], qr[RPT][4], g[RPT][4];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = i0 + r;
    if constexpr (kF32) {
      ldv<4>(rk + i * RAW_LD + d0, kr[r]);
      ldv<4>(rq + i * RAW_LD + d0, qr[r]);
    } else {
      lds_bf16x4(rk + i * RAW_LD + d0 / 2, kr[r]);
      lds_bf16x4(rq + i * RAW_LD + d0 / 2, qr[r]);
    }
    ldv<4>(sG + i * LDK + d0, g[r]);
    if (i >= valid) {
#pragma unroll
      for (int c = 0; c < 4; ++c) g[r][c] = 1.f;
    }
  }
  // ---- log a, summed down this thread's rows
#pragma unroll
  for (int r = 0; r < RPT; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) g[r][c] = logf(g[r][c]) + (r ? g[r - 1][c] : 0.f);
  st4(sTot + rg * DK + d0, g[RPT - 1][0], g[RPT - 1][1], g[RPT - 1][2], g[RPT - 1][3]);
  if (rg == 0) st4(sRow0 + d0, g[0][0], g[0][1], g[0][2], g[0][3]);
  // ---- the q/k L2 norm over each row (QPR lanes), rounded to the io dtype
  if (p.flags & GDN_QK_L2NORM) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      float sk = 0.f, sq = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sk = fmaf(kr[r][c], kr[r][c], sk);
        sq = fmaf(qr[r][c], qr[r][c], sq);
      }
#pragma unroll
      for (int o = QPR / 2; o >= 1; o >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float ik = rsqrtf(sk + kQkNormEps), iq = rsqrtf(sq + kQkNormEps);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kr[r][c] = to_f32(from_f32<T>(kr[r][c] * ik));
        qr[r][c] = to_f32(from_f32<T>(qr[r][c] * iq));
      }
    }
  }
  __syncthreads();
  // ---- G = the thread's running sums plus the row groups above; G_0, G_C
  float off[4] = {0.f, 0.f, 0.f, 0.f}, gc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < RG; ++j) {
    const float4 t = lds4(sTot + j * DK + d0);
    const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (j < rg) off[c] += tv[c];
      gc[c] += tv[c];
    }
  }
  float mid[4];
  bool wide = false;
  {
    const float4 g0 = lds4(sRow0 + d0);
    const float g0v[4] = {g0.x, g0.y, g0.z, g0.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mid[c] = 0.5f * (g0v[c] + gc[c]);
      wide |= !(g0v[c] - gc[c] <= kFactorRange);
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) g[r][c] += off[c];
  const bool factored = !__syncthreads_or(wide);
  // ---- the decayed operands: factored ones to shared memory (K^ over K, K~
  // over G, Q~ over Q, e^m per channel) or the plain K, Q, G;
  // (K o e^{G_C - G})^T and e^{G_C} to the workspace
  const size_t w = (size_t)slot * H + h;
  float* kht = p.ws.KhT + w * C * DK;
  float* sEm = sm + PL::MID;                       // [DK] e^m of a factored chunk
  float* sEc = sEm + DK;                           // [DK] e^{G_C - m} of a factored chunk
  float* sGc = sEc + DK;                           // [DK] G_C
  if (factored) {
    float em[4], ec[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      em[c] = expf(mid[c]);
      ec[c] = expf(gc[c] - mid[c]);
    }
    if (rg == 0) {
      st4(sEm + d0, em[0], em[1], em[2], em[3]);
      st4(sEc + d0, ec[0], ec[1], ec[2], ec[3]);
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      float kt[4], kc[4], qt[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float x = g[r][c] - mid[c];
        const float ex = expf(x), fx = expf(-x);
        kt[c] = kr[r][c] * ex;
        kc[c] = kr[r][c] * fx;
        qt[c] = qr[r][c] * ex;
      }
      const int i = i0 + r;
      st4(sK + i * LDK + d0, kc[0], kc[1], kc[2], kc[3]);
      st4(sG + i * LDK + d0, kt[0], kt[1], kt[2], kt[3]);
      st4(sQ + i * LDK + d0, qt[0], qt[1], qt[2], qt[3]);
    }
  } else {
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = i0 + r;
      st4(sK + i * LDK + d0, kr[r][0], kr[r][1], kr[r][2], kr[r][3]);
      st4(sQ + i * LDK + d0, qr[r][0], qr[r][1], qr[r][2], qr[r][3]);
      st4(sG + i * LDK + d0, g[r][0], g[r][1], g[r][2], g[r][3]);
    }
  }
  if (rg == 0) {
    st4(sGc + d0, gc[0], gc[1], gc[2], gc[3]);
    st4(p.ws.EGC + w * DK + d0, expf(gc[0]), expf(gc[1]), expf(gc[2]), expf(gc[3]));
  }
  __syncthreads();
  // ---- (K o e^{G_C - G})^T to the workspace ([dk][C]), stores coalesced
  // along the chunk's rows: K^ e^{G_C - m} (factored) or K e^{G_C - G}
  for (int e = tid; e < DK * C; e += THREADS) {
    const int d = e / C, i = e % C;
    const float kv = sK[i * LDK + d];
    kht[e] = factored ? kv * sEc[d] : kv * expf(sGc[d] - sG[i * LDK + d]);
  }
  // ---- A and P
  if (factored) ap_factored<DK, PL>(sm, tid);
  else ap_exact<DK, PL>(sm, tid);
  __syncthreads();
  // ---- T = (I + A)^{-1} by 16 x 16 blocks
  solve_blocked(sm + PL::A, sT, sm + PL::SX, tid);
  // ---- a chunk decayed term by term: K o e^G over G, Q o e^G over Q (a
  // factored one keeps K~ and Q~, and its e^m scales W's and Q''s columns);
  // T diag(b) over T
  if (!factored) {
#pragma unroll 4
    for (int e = tid; e < C * DK / 4; e += THREADS) {
      const int i = e / (DK / 4), d = 4 * (e % (DK / 4));
      const float4 gg = lds4(sG + i * LDK + d), kk = lds4(sK + i * LDK + d), qq = lds4(sQ + i * LDK + d);
      const float e0 = expf(gg.x), e1 = expf(gg.y), e2 = expf(gg.z), e3 = expf(gg.w);
      st4(sG + i * LDK + d, kk.x * e0, kk.y * e1, kk.z * e2, kk.w * e3);
      st4(sQ + i * LDK + d, qq.x * e0, qq.y * e1, qq.z * e2, qq.w * e3);
    }
  }
#pragma unroll 4
  for (int e = tid; e < C * C / 4; e += THREADS) {
    const int i = e / (C / 4), j = 4 * (e % (C / 4));
    const float4 t = lds4(sT + i * LDC + j), b = lds4(sb + j);
    st4(sT + i * LDC + j, t.x * b.x, t.y * b.y, t.z * b.z, t.w * b.w);
  }
  __syncthreads();
  // Products with a lower-triangular left factor (T diag(b) or P): thread rows
  // r0 .. r0 + 3 of the 8-row band `band`, columns 64 q + 4 cg ..; warp w takes
  // band w (w < 4) or 11 - w, so the two warps of each scheduler share out the
  // triangle evenly.
  const int wp = tid >> 5, lane = tid & 31;
  const int band = (wp < 4) ? wp : 11 - wp;
  const int r0 = 8 * band + 4 * (lane >> 4), cg = lane & 15, kend = 8 * band + 8;
  const float* sP = sm + PL::P;
  // ---- W = T diag(b) (K o e^G) (factored: (T diag(b) K~) e^m), over K^
  // (its readers, the products, are done)
  {
    float acc[4][DK / 16];
    tri_times<DK / 64>(acc, sT + r0 * LDC, sG, LDK, cg, kend);
    float* gw = p.ws.W + w * C * DK;
#pragma unroll
    for (int q = 0; q < DK / 64; ++q) {
      const float4 em = factored ? lds4(sEm + 64 * q + 4 * cg) : make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float* a = acc[i] + 4 * q;
        a[0] *= em.x;
        a[1] *= em.y;
        a[2] *= em.z;
        a[3] *= em.w;
        st4(sK + (r0 + i) * LDK + 64 * q + 4 * cg, a[0], a[1], a[2], a[3]);
        st4(gw + (r0 + i) * DK + 64 * q + 4 * cg, a[0], a[1], a[2], a[3]);
      }
    }
  }
  __syncthreads();
  // ---- Q' = Q o e^G - P W
  {
    float acc[4][DK / 16];
    tri_times<DK / 64>(acc, sP + r0 * LDC, sK, LDK, cg, kend);
    float* gq = p.ws.Qp + w * C * DK;
#pragma unroll
    for (int q = 0; q < DK / 64; ++q) {
      const float4 em = factored ? lds4(sEm + 64 * q + 4 * cg) : make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 qg = lds4(sQ + (r0 + i) * LDK + 64 * q + 4 * cg);
        st4(gq + (r0 + i) * DK + 64 * q + 4 * cg, fmaf(qg.x, em.x, -acc[i][4 * q]),
            fmaf(qg.y, em.y, -acc[i][4 * q + 1]), fmaf(qg.z, em.z, -acc[i][4 * q + 2]),
            fmaf(qg.w, em.w, -acc[i][4 * q + 3]));
      }
    }
  }
  // ---- per 64 columns of v (staged two blocks deep; block 0 came with q, k
  // and a): U~ = T diag(b) V (V as fp32 over A, U~ over G), then O~ = P U~
  float* sVb = sm + PL::A;
  float* sUb = sG;
  float* gut = p.ws.Ut + w * C * (size_t)p.dv;
  float* got = p.ws.Ot + w * C * (size_t)p.dv;
  for (int vb = 0, buf = 0; vb < p.dv; vb += 64, buf ^= 1) {
    if (vb + 64 < p.dv) stage_v(vb + 64, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();                            // this block's rows
    __syncthreads();                               // and the last block's readers are done
#pragma unroll 4
    for (int e = tid; e < C * 16; e += THREADS) {
      const int i = e >> 4, c = 4 * (e & 15);
      const float* raw = sm + PL::VST + buf * C * 64 + i * VROW;
      float x[4];
      if constexpr (kF32) ldv<4>(raw + c, x);
      else lds_bf16x4(raw + c / 2, x);
      st4(sVb + i * LDC + c, x[0], x[1], x[2], x[3]);
    }
    __syncthreads();
    {
      float acc[4][4];
      tri_times<1>(acc, sT + r0 * LDC, sVb, LDC, cg, kend);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        st4(sUb + (r0 + i) * LDC + 4 * cg, acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        st4(gut + (size_t)(r0 + i) * p.dv + vb + 4 * cg, acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      }
    }
    __syncthreads();
    {
      float acc[4][4];
      tri_times<1>(acc, sP + r0 * LDC, sUb, LDC, cg, kend);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        st4(got + (size_t)(r0 + i) * p.dv + vb + 4 * cg, acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
  }
}

// Warp-level m16n8k8 tf32 MMA (fp32 accumulate) with each operand split into
// a tf32 high part and a tf32 remainder: a b ~= ah bh + ah bl + al bh, the
// three partial products in separate accumulators, which keeps the products
// close to fp32.
__device__ __forceinline__ uint32_t tf32_hi(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo) {
  hi = tf32_hi(x);
  lo = tf32_hi(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// A chain's state slice of NV = 16 columns and the chunk's operands.  W, Q'
// (by chunk parity) and (K o e^{G_C - G})^T arrive as TMA boxes of 32 fp32
// columns in the 128-byte swizzle (element (r, k) of a box at row r, 16-byte
// chunk (k / 4) xor (r % 8)), which keeps the fragment reads conflict-free;
// the state and U are padded rows (B fragments, banks 24 q + g).
template <int DK>
struct ChainPlan {
  static constexpr int NV = 16;
  static constexpr int LDS = NV + 8;
  static constexpr int TILE = C * DK;              // floats of one W, Q' or K^T tile
  static constexpr int W = 0;                      // 2 tiles, by chunk parity: DK / 32 boxes of [C][32]
  static constexpr int QP = W + 2 * TILE;          // 2 tiles
  static constexpr int KT = QP + 2 * TILE;         // C / 32 boxes of [DK][32]
  static constexpr int SIG = KT + TILE;            // [DK][LDS]
  static constexpr int SIGH = SIG + DK * LDS;      // [DK][LDS] the state split once per chunk: tf32 high part
  static constexpr int SIGL = SIGH + DK * LDS;     // [DK][LDS] and remainder (the B operand of the state pass)
  static constexpr int U = SIGL + DK * LDS;        // [C][LDS]  U's tf32 high part (the carry's B operand)
  static constexpr int UL = U + C * LDS;           // [C][LDS]  and remainder
  static constexpr int UT = UL + C * LDS;          // [C][LDS]  U~ slice
  static constexpr int OT = UT + C * LDS;          // [C][LDS]  O~ slice
  static constexpr int EGC = OT + C * LDS;         // [DK]      e^{G_C}
  static constexpr int BAR = EGC + DK;             // mbarriers: W / Q' by parity, K^T; abort flag
  static constexpr int FLOATS = BAR + 8;
  static constexpr size_t BYTES = (size_t)FLOATS * 4 + 1024;   // + alignment of the base to 1024 bytes
};
static_assert(ChainPlan<128>::BYTES <= 232448, "KDA chain shared memory");
static_assert(ChainPlan<128>::TILE % 256 == 0 && ChainPlan<64>::TILE % 256 == 0, "1024-byte tile alignment");

// Element (r, k) of a swizzled tile of boxes [rows][32] (box = k / 32).
template <int ROWS>
__device__ __forceinline__ float sw_at(const float* tile, int r, int k) {
  return tile[(k >> 5) * ROWS * 32 + r * 32 + ((((k & 31) >> 2) ^ (r & 7)) << 2) + (k & 3)];
}

// acc[nt] += A (16 x 8 at rows m0.., k-step k0, A read through `a_at` and
// split here) times B (8 x 16, element (k, n) at [k * LDB + n], already split
// into tf32 high parts BH and remainders BL), fragments of lane (g, q).
template <int LDB, typename AAt>
__device__ __forceinline__ void mma_step_split(float (&acc)[2][3][4], AAt a_at, const uint32_t* BH, const uint32_t* BL,
                                               int k0, int g, int q) {
  uint32_t ah[4], al[4];
  tf32_split(a_at(g, k0 + q), ah[0], al[0]);
  tf32_split(a_at(g + 8, k0 + q), ah[1], al[1]);
  tf32_split(a_at(g, k0 + q + 4), ah[2], al[2]);
  tf32_split(a_at(g + 8, k0 + q + 4), ah[3], al[3]);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int o0 = (k0 + q) * LDB + 8 * nt + g, o1 = o0 + 4 * LDB;
    const uint32_t bh[2] = {BH[o0], BH[o1]}, bl[2] = {BL[o0], BL[o1]};
    mma_16x8x8(acc[nt][0], ah, bh);
    mma_16x8x8(acc[nt][1], ah, bl);
    mma_16x8x8(acc[nt][2], al, bh);
  }
}

__device__ __forceinline__ void kda_tma_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void kda_bulk(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// One CTA per (sequence, head, 16-column dv slice): the chain through its
// chunks, operands from the workspace, both products on the tensor cores
// (3xTF32 MMAs, fp32 accumulate).  [W; Q'] Sigma_0: warp w takes 16 rows of W
// (w < 4, giving U) or of Q' (w >= 4, giving O); the carry
// (K o e^{G_C - G})^T U: warp w takes state rows 16 w .. 16 w + 15.  Each
// output element belongs to one lane, so there is nothing to reduce.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1)
    gdn_prefill_kda_chain_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                                 const __grid_constant__ CUtensorMap tm_kt, const Params p) {
  using PL = ChainPlan<DK>;
  constexpr int NV = PL::NV, LDS = PL::LDS, TILE = PL::TILE;
  extern __shared__ __align__(16) unsigned char smraw[];
  float* sm = reinterpret_cast<float*>(smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u));
  float* sW = sm + PL::W;
  float* sQp = sm + PL::QP;
  float* sKt = sm + PL::KT;
  float* sSig = sm + PL::SIG;
  uint32_t* sSigH = reinterpret_cast<uint32_t*>(sm + PL::SIGH);
  uint32_t* sSigL = reinterpret_cast<uint32_t*>(sm + PL::SIGL);
  uint32_t* sUH = reinterpret_cast<uint32_t*>(sm + PL::U);
  uint32_t* sUL = reinterpret_cast<uint32_t*>(sm + PL::UL);
  float* sUt = sm + PL::UT;
  float* sOt = sm + PL::OT;
  float* sEGC = sm + PL::EGC;
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(sm + PL::BAR);   // [2], W and Q' by buffer
  uint64_t* bar_k = bar_w + 2;                                    // the carry's operands
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_w + 3);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int n_slices = p.dv / NV;
  const int slice = blockIdx.x % n_slices;
  const int chain = blockIdx.x / n_slices;
  const int h = chain % p.H;
  const int seq = chain / p.H;
  const int H = p.H, dv = p.dv;
  int t0, t1;
  seq_range(p, seq, t0, t1, tid == 0);
  const int n_chunks = (t1 - t0 + C - 1) / C;
  const long long slot0 = slot_base(seq, t0);
  const int col0 = slice * NV;
  const size_t sbase = ((size_t)seq * H + h) * DK * (size_t)dv + col0;
  T* o = static_cast<T*>(p.o);

  // Thread 0 issues W and Q' of chunk c (into buffer c & 1) and the carry's
  // (K o e^{G_C - G})^T and e^{G_C}, each after the barrier that ends its
  // buffer's last reader; the U~ and O~ slices are one cp.async group per
  // chunk (empty past the last chunk).
  int issued_w0 = 0, issued_w1 = 0, issued_k = 0;  // thread 0's count of each barrier's phases
  auto issue_w = [&](int c) {
    const int y = (int)(((slot0 + c) * H + h) * C);
    uint64_t* bar = &bar_w[c & 1];
    mbar_arrive_expect_tx(bar, 2 * TILE * 4);
#pragma unroll
    for (int b = 0; b < DK / 32; ++b) {
      kda_tma_2d(sW + (c & 1) * TILE + b * C * 32, &tm_w, bar, 32 * b, y);
      kda_tma_2d(sQp + (c & 1) * TILE + b * C * 32, &tm_q, bar, 32 * b, y);
    }
    if (c & 1) ++issued_w1;
    else ++issued_w0;
  };
  auto issue_k = [&](int c) {
    const size_t w = (size_t)(slot0 + c) * H + h;
    mbar_arrive_expect_tx(bar_k, (TILE + DK) * 4);
#pragma unroll
    for (int b = 0; b < C / 32; ++b) kda_tma_2d(sKt + b * DK * 32, &tm_kt, bar_k, 32 * b, (int)(w * DK));
    kda_bulk(sEGC, p.ws.EGC + w * DK, DK * 4, bar_k);
    ++issued_k;
  };
  auto load_u = [&](int c) {
    if (c < n_chunks) {
      const size_t base = ((size_t)(slot0 + c) * H + h) * C * (size_t)dv + col0;
      for (int e = tid; e < 2 * C * (NV / 4); e += THREADS) {
        const int m = e / (C * (NV / 4)), r = e % (C * (NV / 4));
        const int i = r / (NV / 4), c4 = r % (NV / 4);
        cp_async16((m ? sOt : sUt) + i * LDS + 4 * c4, (m ? p.ws.Ot : p.ws.Ut) + base + (size_t)i * dv + 4 * c4);
      }
    }
    cp_async_commit();
  };

  if (tid == 0) {
    mbar_init(&bar_w[0], 1);
    mbar_init(&bar_w[1], 1);
    mbar_init(bar_k, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && n_chunks > 0) issue_w(0);
  load_u(0);
  for (int e = tid; e < DK * NV; e += THREADS) {
    const int d = e / NV, c = e % NV;
    const float x = p.S0 ? p.S0[sbase + (size_t)d * dv + c] : 0.f;
    sSig[d * LDS + c] = x;
    tf32_split(x, sSigH[d * LDS + c], sSigL[d * LDS + c]);
  }
  // Every wait is bounded: a timeout records GDN_ERR_TIMEOUT, raises the
  // abort flag, and the block leaves the loop at the next barrier.
  for (int c = 0; c < n_chunks; ++c) {
    const int tok0 = t0 + c * C, valid = min(C, t1 - tok0);
    const bool okw = mbar_wait_bounded(&bar_w[c & 1], (c >> 1) & 1, abort_flag, p.status);
    cp_async_wait<0>();                            // the U~ and O~ slices
    if (__syncthreads_or(!okw || *abort_flag != 0)) break;
    if (tid == 0) {
      fence_proxy_async_smem();                    // the last generic reads of the refilled buffers come first
      issue_k(c);
      if (c + 1 < n_chunks) issue_w(c + 1);
    }
    // ---- U = U~ - W Sigma_0 (warps 0-3) and O = scale (Q' Sigma_0 + O~)
    // with the output gate and the loop residual (warps 4-7)
    {
      const int r0 = 16 * (warp & 3);
      const float* At = ((warp < 4) ? sW : sQp) + (c & 1) * TILE;
      auto a_at = [&](int m, int k) { return sw_at<C>(At, r0 + m, k); };
      float acc[2][3][4] = {};
#pragma unroll 4
      for (int k0 = 0; k0 < DK; k0 += 8) mma_step_split<LDS>(acc, a_at, sSigH, sSigL, k0, g, q);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int row = r0 + g + 8 * hf, col = 8 * nt + 2 * q;
          const float x0 = acc[nt][0][2 * hf] + (acc[nt][1][2 * hf] + acc[nt][2][2 * hf]);
          const float x1 = acc[nt][0][2 * hf + 1] + (acc[nt][1][2 * hf + 1] + acc[nt][2][2 * hf + 1]);
          if (warp < 4) {
            const float2 ut = *reinterpret_cast<const float2*>(sUt + row * LDS + col);
            uint2 uh, ul;
            tf32_split(ut.x - x0, uh.x, ul.x);
            tf32_split(ut.y - x1, uh.y, ul.y);
            *reinterpret_cast<uint2*>(sUH + row * LDS + col) = uh;
            *reinterpret_cast<uint2*>(sUL + row * LDS + col) = ul;
          } else if (row < valid) {
            const float2 ot = *reinterpret_cast<const float2*>(sOt + row * LDS + col);
            const float og = p.gate ? 1.f / (1.f + __expf(-p.gate[(size_t)(tok0 + row) * H + h])) : 1.f;
            const float sv[2] = {x0 + ot.x, x1 + ot.y};
            const size_t obase = ((size_t)(tok0 + row) * H + h) * dv + col0 + col;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float y = p.scale * sv[j];
              if (p.gate) y *= og;
              if (p.h_prev) {
                const float hp = to_f32(static_cast<const T*>(p.h_prev)[obase + j]);
                y = fmaf(p.rho[(size_t)h * dv + col0 + col + j], hp, to_f32(from_f32<T>(y)));
              }
              o[obase + j] = from_f32<T>(y);
            }
          }
        }
    }
    const bool okk = mbar_wait_bounded(bar_k, c & 1, abort_flag, p.status);
    if (__syncthreads_or(!okk || *abort_flag != 0)) break;
    load_u(c + 1);
    // ---- Sigma_C = Diag(e^{G_C}) Sigma_0 + (K o e^{G_C - G})^T U
    if (16 * warp < DK) {
      const int d0 = 16 * warp;
      auto a_at = [&](int m, int k) { return sw_at<DK>(sKt, d0 + m, k); };
      float acc[2][3][4] = {};
#pragma unroll
      for (int k0 = 0; k0 < C; k0 += 8) mma_step_split<LDS>(acc, a_at, sUH, sUL, k0, g, q);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int d = d0 + g + 8 * hf, col = 8 * nt + 2 * q;
          const float x0 = acc[nt][0][2 * hf] + (acc[nt][1][2 * hf] + acc[nt][2][2 * hf]);
          const float x1 = acc[nt][0][2 * hf + 1] + (acc[nt][1][2 * hf + 1] + acc[nt][2][2 * hf + 1]);
          float2* sg = reinterpret_cast<float2*>(sSig + d * LDS + col);
          const float2 old = *sg;
          const float gd = sEGC[d];
          const float2 nw = make_float2(fmaf(gd, old.x, x0), fmaf(gd, old.y, x1));
          *sg = nw;
          uint2 sh, sl;
          tf32_split(nw.x, sh.x, sl.x);
          tf32_split(nw.y, sh.y, sl.y);
          *reinterpret_cast<uint2*>(sSigH + d * LDS + col) = sh;
          *reinterpret_cast<uint2*>(sSigL + d * LDS + col) = sl;
        }
    }
  }
  // leave no copy in flight: the last phase issued on each barrier
  if (tid == 0) {
    if (issued_w0 > 0) mbar_wait_bounded(&bar_w[0], (issued_w0 - 1) & 1, nullptr, p.status);
    if (issued_w1 > 0) mbar_wait_bounded(&bar_w[1], (issued_w1 - 1) & 1, nullptr, p.status);
    if (issued_k > 0) mbar_wait_bounded(bar_k, (issued_k - 1) & 1, nullptr, p.status);
  }
  cp_async_wait<0>();
  __syncthreads();
  if (p.S_T && *abort_flag == 0) {
    for (int e = tid; e < DK * NV; e += THREADS) {
      const int d = e / NV, c = e % NV;
      p.S_T[sbase + (size_t)d * dv + c] = sSig[d * LDS + c];
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

template <int DK, typename T>
static cudaError_t launch_two(const Params& kp, long long chunk_blocks, long long chain_blocks,
                              cudaStream_t stream) {
  static std::atomic<bool> set_prep[kMaxDevices], set_chain[kMaxDevices];
  constexpr size_t prep_bytes = PrepPlan<DK>::BYTES;
  constexpr size_t chain_bytes = ChainPlan<DK>::BYTES;
  // W, Q' as [slots * H * C][dk] and (K o e^{G_C - G})^T as [slots * H * dk][C],
  // fp32, boxes of 32 columns x C or dk rows in the 128-byte swizzle
  const long long sh = kp.ws.n_slots * kp.H;
  CUtensorMap mw, mq, mk;
  if (!make_map_2d(&mw, kp.ws.W, DK, sh * C, 32, C, 4) || !make_map_2d(&mq, kp.ws.Qp, DK, sh * C, 32, C, 4) ||
      !make_map_2d(&mk, kp.ws.KhT, C, sh * DK, 32, DK, 4))
    return cudaErrorInvalidValue;
  cudaError_t e = smem_attr_once(set_prep, gdn_prefill_kda_prep_kernel<DK, T>, prep_bytes);
  if (e == cudaSuccess) e = smem_attr_once(set_chain, gdn_prefill_kda_chain_kernel<DK, T>, chain_bytes);
  if (e != cudaSuccess) return e;
  gdn_prefill_kda_prep_kernel<DK, T><<<(unsigned)chunk_blocks, THREADS, prep_bytes, stream>>>(kp);
  gdn_prefill_kda_chain_kernel<DK, T><<<(unsigned)chain_blocks, THREADS, chain_bytes, stream>>>(mw, mq, mk, kp);
  return cudaGetLastError();
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static long long n_slots(const gdn_fwd_params* p) { return (long long)p->total_tokens / C + p->n_seq + 1; }

}  // namespace kda

// Bytes of the two-launch schedule's workspace: W, Q' and K o e^{G_C - G}
// ([slots][H][C][dk] fp32 each), U~ and O~ ([slots][H][C][dv]) and e^{G_C}
// ([slots][H][dk]).
size_t prefill_kda_workspace(const gdn_fwd_params* p) {
  const size_t sh = (size_t)kda::n_slots(p) * p->H;
  const size_t dk = (size_t)p->dk, dv = (size_t)p->dv, c = kda::C;
  return 3 * kda::align256(sh * c * dk * 4) + 2 * kda::align256(sh * c * dv * 4) + kda::align256(sh * dk * 4);
}

gdn_status launch_prefill_kda(const gdn_fwd_params* p, unsigned* status, void* ws, cudaStream_t stream) {
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
  kp.ws = kda::Ws{};
  const long long chains = (long long)p->n_seq * p->H;
  if (chains <= 0) return GDN_OK;
  cudaError_t e;
  if (ws) {
    // two launches: the chunks' operands, then the chains
    const long long n_slots = kda::n_slots(p);
    const size_t sh = (size_t)n_slots * p->H;
    const size_t dk = (size_t)p->dk, c = kda::C;
    char* w = static_cast<char*>(ws);
    float** rows_dk[] = {&kp.ws.W, &kp.ws.Qp, &kp.ws.KhT};
    for (float** a : rows_dk) {
      *a = reinterpret_cast<float*>(w);
      w += kda::align256(sh * c * dk * 4);
    }
    float** rows_dv[] = {&kp.ws.Ut, &kp.ws.Ot};
    for (float** a : rows_dv) {
      *a = reinterpret_cast<float*>(w);
      w += kda::align256(sh * c * (size_t)p->dv * 4);
    }
    kp.ws.EGC = reinterpret_cast<float*>(w);
    kp.ws.n_slots = n_slots;
    const long long chunk_blocks = n_slots * p->H;
    const long long chain_blocks = chains * (p->dv / 16);   // 16 columns per chain CTA
    if (chunk_blocks > 0x7fffffffLL || chain_blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (p->io_dtype == GDN_BF16)
      e = p->dk == 128 ? kda::launch_two<128, __nv_bfloat16>(kp, chunk_blocks, chain_blocks, stream)
                       : kda::launch_two<64, __nv_bfloat16>(kp, chunk_blocks, chain_blocks, stream);
    else
      e = p->dk == 128 ? kda::launch_two<128, float>(kp, chunk_blocks, chain_blocks, stream)
                       : kda::launch_two<64, float>(kp, chunk_blocks, chain_blocks, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }
  const long long blocks = chains * kp.n_slices;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  if (p->io_dtype == GDN_BF16)
    e = p->dk == 128 ? kda::launch_t<128, __nv_bfloat16>(kp, blocks, stream)
                     : kda::launch_t<64, __nv_bfloat16>(kp, blocks, stream);
  else
    e = p->dk == 128 ? kda::launch_t<128, float>(kp, blocks, stream)
                     : kda::launch_t<64, float>(kp, blocks, stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
