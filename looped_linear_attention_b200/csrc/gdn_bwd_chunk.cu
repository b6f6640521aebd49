// Chunkwise reverse mode of the gated delta rule (gdn_chunk_bwd, default
// path).  The forward recurrence ("LT2: Linear-Time Looped Transformers", §2,
// in the dk x dv orientation S_t = a_t (S_{t-1} - b_t k_t x_t^T) + b_t k_t v_t^T,
// x_t = S_{t-1}^T k_t, o_t = scale S_t^T q_t) in its chunked form: for a chunk
// of C = 64 tokens with start state S, g_i = sum_{m <= i} log a_m (within the
// chunk), gamma_i = e^{g_i}, D_ij = e^{g_i - g_j} (i >= j), r_i = e^{g_C - g_i}
// (g_C = g of the last row):
//     A_ij = b_i D_ij k_i.k_j (i > j),  T = (I + A)^{-1},
//     R = diag(b) V - diag(b gamma) K S,  U = T R,
//     P_ij = scale D_ij q_i.k_j (i >= j),
//     O = scale diag(gamma) Q S + P U,
//     S_end = gamma_C S + (diag(r) K)^T U.
// With W = T diag(b gamma) K, U~ = T diag(b) V and Qh = scale diag(gamma) Q -
// P W, the chunk maps (S -> S_end, O) as S_end = M S + (diag(r)K)^T U~ with
// M = gamma_C I - (diag(r)K)^T W, and O = Qh S + P U~.  Its reverse mode, given
// dO and dE = dloss/dS_end:
//     dU  = P^T dO + diag(r) K dE,     dR = T^T dU,
//     dS  = gamma_C dE + Qh^T dO - W^T (diag(r) K dE)   (= M^T dE + Qh^T dO)
//     dV  = diag(b) dR,                dA = -strictly_lower(dR U^T),
//     dP  = lower(dO U^T),
//     dq  = scale diag(gamma) dO S^T + (dP o scale D) K,
//     dk  = -diag(b gamma) dR S^T + diag(r) U dE^T + (A' + A'^T) K + (dP o scale D)^T Q,
//           with A'_ij = dA_ij b_i D_ij,
//     db_i = dR_i.(v_i - gamma_i (K S)_i) + sum_{j<i} dA_ij D_ij k_i.k_j,
// and for the log-decays (each term's derivative through the D, gamma and r
// factors it contains): dg_i collects
//     scale gamma_i dO_i.(S^T q_i)  -  b_i gamma_i dR_i.(S^T k_i)
//   + sum_j (dP o P)_ij - sum_j (dP o P)_ji + sum_j (dA o A)_ij - sum_j (dA o A)_ji
//   - kappa_i,  kappa_i = r_i U_i.(dE^T k_i),
// and the last row also sum_i kappa_i + gamma_C <dE, S>; then
// dlog a_m = sum_{i >= m} dg_i and grad_a_m = dlog a_m / a_m.
//
// Launches (fp32 on the CUDA cores, register-tiled products from shared memory):
//   1. gdn_bwd_prep_kernel    one CTA per (chunk, head): T, W, U~, Qh, g
//   2. gdn_bwd_states_kernel  one CTA per (sequence, head, 32 columns of dv):
//                             the chunk start states S_c, forward in order
//   3. gdn_bwd_dstates_kernel the same grid: dE_c backwards, and grad_S0
//   4. gdn_bwd_grads_kernel   one CTA per (chunk, head): every gradient of the
//                             chunk's tokens from S_c and dE_c
// Chunks of sequence s take workspace slots t0_s / C + 2 s + c (consecutive
// sequences' first slots differ by at least their chunk count plus one).
#include "common.cuh"

namespace gdn {
namespace cbwd {

constexpr int C = 64;
constexpr int THREADS = 256;
constexpr int NS = 32;            // dv columns per tile (grads) and per state-pass CTA
constexpr int LDT = NS + 1;       // row stride of [rows][NS] tiles
constexpr int LDC = C + 1;        // row stride of C x C tiles
constexpr float kMinGate = 1e-30f;   // a is clamped to this before its logarithm

struct KParams {
  const void *q, *k, *v, *go;
  const float *a, *b, *S0, *gST;
  float *gq, *gk, *gv, *ga, *gb, *gS0;
  const int32_t* cu;
  int n_seq, seq_len, total, H, dv;
  float scale;
  long long n_slots;                // chunk slots per head
  float *W, *Ut, *Qh, *G;           // per (slot, head): [C][dk], [C][dv], [C][dk], [C]
  float *Sst, *dE;                  // per (slot, head): [dk][dv]
  unsigned* status;
};

__device__ __forceinline__ float ldx(const float* p, size_t i) { return __ldg(p + i); }
__device__ __forceinline__ float ldx(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

// Token range of sequence s, clamped to [0, total] (invalid offsets reported).
__device__ __forceinline__ void seq_range(const KParams& p, int s, int& t0, int& t1, bool report) {
  if (p.cu) {
    t0 = __ldg(p.cu + s);
    t1 = __ldg(p.cu + s + 1);
  } else {
    t0 = s * p.seq_len;
    t1 = t0 + p.seq_len;
  }
  const int c0 = min(max(t0, 0), p.total);
  const int c1 = min(max(t1, c0), p.total);
  if (report && (c0 != t0 || c1 != t1)) record_status(p.status, GDN_ERR_INVALID);
  t0 = c0;
  t1 = c1;
}
__device__ __forceinline__ long long slot_base(int s, int t0) { return t0 / C + 2LL * s; }

// Slot -> (sequence, chunk): the last sequence whose first slot is <= slot;
// false when the slot holds no chunk.
__device__ bool slot_chunk(const KParams& p, long long slot, int& s, int& c, int& t0, int& n) {
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
  const long long cc = slot - slot_base(lo, s0);
  const int n_chunks = (s1 - s0 + C - 1) / C;
  if (cc < 0 || cc >= n_chunks) return false;
  s = lo;
  c = (int)cc;
  t0 = s0 + c * C;
  n = min(C, s1 - t0);
  return true;
}

// acc[i][j] += sum_k A(i, k) B(k, j) over k < K for a thread's TM x TN tile;
// fa(i, k) and fb(k, j) read the operands.
template <int TM, int TN, int K, class FA, class FB>
__device__ __forceinline__ void gemm(float (&acc)[TM][TN], FA fa, FB fb) {
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float av[TM], bv[TN];
#pragma unroll
    for (int i = 0; i < TM; ++i) av[i] = fa(i, k);
#pragma unroll
    for (int j = 0; j < TN; ++j) bv[j] = fb(k, j);
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}
template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// Sum over the 16 threads that share tid / 16 (one half-warp).
__device__ __forceinline__ float half_warp_sum(float x) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Chunk gate vectors (threads 0-63, one row each): g, gamma, b, r, a.
struct Vec {
  float *g, *gam, *b, *r, *a;
};
__device__ __forceinline__ void chunk_gates(const KParams& p, int t0, int n, int h, Vec V, float* s_carry,
                                            int tid) {
  float la = 0.f, bb = 0.f, aa = 1.f;
  if (tid < C) {
    if (tid < n) {
      const size_t ti = (size_t)(t0 + tid) * p.H + h;
      aa = __ldg(p.a + ti);
      bb = __ldg(p.b + ti);
      la = logf(fmaxf(aa, kMinGate));
    }
    const int lane = tid & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, la, off);
      if (lane >= off) la += y;
    }
    if (tid == 31) *s_carry = la;
  }
  __syncthreads();
  if (tid < C) {
    if (tid >= 32) la += *s_carry;
    V.g[tid] = la;
    V.gam[tid] = expf(la);
    V.b[tid] = bb;
    V.a[tid] = aa;
  }
  __syncthreads();
  if (tid < C) V.r[tid] = expf(V.g[C - 1] - V.g[tid]);
}

// Rows [0, n) of a [tokens][H][width] input into shared memory ([C][ld]
// fp32, columns [c0, c0 + cols)), zeros below.
template <typename T>
__device__ __forceinline__ void load_rows(float* dst, int ld, const T* src, int t0, int n, int h, int H,
                                          int width, int c0, int cols, int tid) {
  for (int e = tid; e < C * cols; e += THREADS) {
    const int i = e / cols, c = e % cols;
    dst[i * ld + c] = (i < n) ? ldx(src, ((size_t)(t0 + i) * H + h) * width + c0 + c) : 0.f;
  }
}

// T = (I + A)^{-1} with A_ij = b_i KK_ij (i > j): column `col` by forward
// substitution, held in registers, four partial sums per row.
__device__ __forceinline__ void solve_column(const float* sKK, const float* sb, float* sT, int col) {
  float t[C];
#pragma unroll
  for (int i = 0; i < C; ++i) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < i; ++m) acc[m & 3] = fmaf(sKK[i * LDC + m], t[m], acc[m & 3]);
    t[i] = ((i == col) ? 1.f : 0.f) - sb[i] * ((acc[0] + acc[1]) + (acc[2] + acc[3]));
  }
#pragma unroll
  for (int i = 0; i < C; ++i) sT[i * LDC + col] = t[i];
}

// Shared setup of the prep and grads kernels: K and Q rows, gate vectors,
// KK = D o K K^T (strictly lower), P = scale D o Q K^T (lower, diagonal
// included) and T.
template <int DK, typename T>
__device__ __forceinline__ void chunk_setup(const KParams& p, int t0, int n, int h, float* sK, float* sQ,
                                            float* sKK, float* sP, float* sT, Vec V, float* s_carry,
                                            int tid) {
  constexpr int LDK = DK + 1;
  load_rows(sK, LDK, static_cast<const T*>(p.k), t0, n, h, p.H, DK, 0, DK, tid);
  load_rows(sQ, LDK, static_cast<const T*>(p.q), t0, n, h, p.H, DK, 0, DK, tid);
  chunk_gates(p, t0, n, h, V, s_carry, tid);
  __syncthreads();
  {
    // thread: rows r0 .. r0+3, columns cg + 16 j (interleaved: no bank conflicts)
    const int r0 = (tid >> 4) * 4, cg = tid & 15;
    float kk[4][4], qk[4][4];
    zero(kk);
    zero(qk);
    // both products share the B operand K^T (B(k, j) = K[cg + 16 j][k])
#pragma unroll 2
    for (int k = 0; k < DK; ++k) {
      float ak[4], aq[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ak[i] = sK[(r0 + i) * LDK + k];
        aq[i] = sQ[(r0 + i) * LDK + k];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = sK[(cg + 16 * j) * LDK + k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          kk[i][j] = fmaf(ak[i], bv[j], kk[i][j]);
          qk[i][j] = fmaf(aq[i], bv[j], qk[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + i, c = cg + 16 * j;
        const float d = (c <= r) ? expf(V.g[r] - V.g[c]) : 0.f;
        sKK[r * LDC + c] = (c < r) ? d * kk[i][j] : 0.f;
        sP[r * LDC + c] = p.scale * d * qk[i][j];
      }
  }
  __syncthreads();
  if (tid < C) solve_column(sKK, V.b, sT, tid);
  __syncthreads();
}

template <int DK>
struct PrepPlan {
  static constexpr int LDK = DK + 1;
  static constexpr int K = 0;
  static constexpr int Q = K + C * LDK;
  static constexpr int W = Q + C * LDK;
  static constexpr int KK = W + C * LDK;
  static constexpr int P = KK + C * LDC;
  static constexpr int T = P + C * LDC;
  static constexpr int V = T + C * LDC;       // [C][LDT]
  static constexpr int VEC = V + C * LDT;     // 5 x C + carry
  static constexpr int FLOATS = VEC + 5 * C + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

// 1. Per (chunk, head): W = T diag(b gamma) K, U~ = T diag(b) V, Qh = scale
// diag(gamma) Q - P W and g, into the workspace.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_prep_kernel(const KParams p) {
  extern __shared__ float smf[];
  using PL = PrepPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TN = DK / 16;
  const int tid = threadIdx.x;
  const long long slot = blockIdx.x / p.H;
  const int h = blockIdx.x % p.H;
  int s, c, t0, n;
  if (!slot_chunk(p, slot, s, c, t0, n)) return;
  float *sK = smf + PL::K, *sQ = smf + PL::Q, *sW = smf + PL::W, *sKK = smf + PL::KK, *sP = smf + PL::P,
        *sT = smf + PL::T, *sV = smf + PL::V;
  Vec V{smf + PL::VEC, smf + PL::VEC + C, smf + PL::VEC + 2 * C, smf + PL::VEC + 3 * C,
        smf + PL::VEC + 4 * C};
  chunk_setup<DK, T>(p, t0, n, h, sK, sQ, sKK, sP, sT, V, smf + PL::VEC + 5 * C, tid);
  const size_t wsi = (size_t)slot * p.H + h;
  const int r0 = (tid >> 4) * 4;
  {
    // W [C][DK] (thread columns cg + 16 j)
    const int cg = tid & 15;
    float acc[4][TN];
    zero(acc);
    gemm<4, TN, C>(acc, [&](int i, int k) { return sT[(r0 + i) * LDC + k]; },
                   [&](int k, int j) { return V.b[k] * V.gam[k] * sK[k * LDK + cg + 16 * j]; });
    float* gW = p.W + wsi * C * DK;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) {
        sW[(r0 + i) * LDK + cg + 16 * j] = acc[i][j];
        gW[(size_t)(r0 + i) * DK + cg + 16 * j] = acc[i][j];
      }
  }
  if (tid < C) p.G[wsi * C + tid] = V.g[tid];
  __syncthreads();
  {
    // Qh [C][DK] = scale diag(gamma) Q - P W
    const int cg = tid & 15;
    float acc[4][TN];
    zero(acc);
    gemm<4, TN, C>(acc, [&](int i, int k) { return sP[(r0 + i) * LDC + k]; },
                   [&](int k, int j) { return sW[k * LDK + cg + 16 * j]; });
    float* gQ = p.Qh + wsi * C * DK;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j)
        gQ[(size_t)(r0 + i) * DK + cg + 16 * j] =
            p.scale * V.gam[r0 + i] * sQ[(r0 + i) * LDK + cg + 16 * j] - acc[i][j];
  }
  // U~ [C][dv], 32 columns at a time
  float* gU = p.Ut + wsi * C * p.dv;
  for (int col0 = 0; col0 < p.dv; col0 += NS) {
    __syncthreads();
    load_rows(sV, LDT, static_cast<const T*>(p.v), t0, n, h, p.H, p.dv, col0, NS, tid);
    __syncthreads();
    const int c0 = (tid & 15) * 2;
    float acc[4][2];
    zero(acc);
    gemm<4, 2, C>(acc, [&](int i, int k) { return sT[(r0 + i) * LDC + k]; },
                  [&](int k, int j) { return V.b[k] * sV[k * LDT + c0 + j]; });
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) gU[(size_t)(r0 + i) * p.dv + col0 + c0 + j] = acc[i][j];
  }
}

template <int DK>
struct StatePlan {
  static constexpr int LDK = DK + 1;
  static constexpr int S = 0;                  // [DK][LDT]
  static constexpr int W = S + DK * LDT;       // [C][LDK]
  static constexpr int KH = W + C * LDK;       // [C][LDK]  diag(r) K
  static constexpr int QH = KH + C * LDK;      // [C][LDK]  (dstates only)
  static constexpr int X = QH + C * LDK;       // [C][LDT]
  static constexpr int DO = X + C * LDT;       // [C][LDT]  (dstates only)
  static constexpr int VEC = DO + C * LDT;     // g, r
  static constexpr int FLOATS = VEC + 2 * C;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

// Chain (sequence, head) and column slice of a state-pass block.
__device__ __forceinline__ void state_block(const KParams& p, int& s, int& h, int& col0) {
  const int n_cs = p.dv / NS;
  col0 = (blockIdx.x % n_cs) * NS;
  const int chain = blockIdx.x / n_cs;
  s = chain / p.H;
  h = chain % p.H;
}

// Loads of one chunk for the state passes: W (and Qh), diag(r) K, g and r.
template <int DK, typename T>
__device__ __forceinline__ void state_chunk_loads(const KParams& p, size_t wsi, int t0, int n, int h,
                                                  float* sW, float* sQh, float* sKh, float* sg, float* sr,
                                                  int tid) {
  constexpr int LDK = DK + 1;
  if (tid < C) sg[tid] = p.G[wsi * C + tid];
  const float4* gW = reinterpret_cast<const float4*>(p.W + wsi * C * DK);
  const float4* gQ = reinterpret_cast<const float4*>(p.Qh + wsi * C * DK);
  for (int e = tid; e < C * DK / 4; e += THREADS) {
    const int i = (e * 4) / DK, d = (e * 4) % DK;
    const float4 w = gW[e];
    sW[i * LDK + d] = w.x;
    sW[i * LDK + d + 1] = w.y;
    sW[i * LDK + d + 2] = w.z;
    sW[i * LDK + d + 3] = w.w;
    if (sQh) {
      const float4 x = gQ[e];
      sQh[i * LDK + d] = x.x;
      sQh[i * LDK + d + 1] = x.y;
      sQh[i * LDK + d + 2] = x.z;
      sQh[i * LDK + d + 3] = x.w;
    }
  }
  __syncthreads();
  if (tid < C) sr[tid] = expf(sg[C - 1] - sg[tid]);
  __syncthreads();
  const T* k = static_cast<const T*>(p.k);
  for (int e = tid; e < C * DK; e += THREADS) {
    const int i = e / DK, d = e % DK;
    sKh[i * LDK + d] = (i < n) ? sr[i] * ldx(k, ((size_t)(t0 + i) * p.H + h) * DK + d) : 0.f;
  }
}

// 2. Chunk start states, forward: S_c[:, J] into the workspace, then
// S <- gamma_C S + (diag(r) K)^T (U~[:, J] - W S).
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_states_kernel(const KParams p) {
  extern __shared__ float smf[];
  using PL = StatePlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TM = DK / 16;
  const int tid = threadIdx.x;
  int s, h, col0;
  state_block(p, s, h, col0);
  int t0, t1;
  seq_range(p, s, t0, t1, tid == 0 && col0 == 0 && h == 0);
  float *sS = smf + PL::S, *sW = smf + PL::W, *sKh = smf + PL::KH, *sX = smf + PL::X;
  float *sg = smf + PL::VEC, *sr = smf + PL::VEC + C;
  const size_t sd = (size_t)DK * p.dv;
  const size_t sb0 = ((size_t)s * p.H + h) * sd;
  for (int e = tid; e < DK * NS; e += THREADS) {
    const int d = e / NS, c = e % NS;
    sS[d * LDT + c] = p.S0 ? p.S0[sb0 + (size_t)d * p.dv + col0 + c] : 0.f;
  }
  const int n_chunks = (t1 - t0 + C - 1) / C;
  const long long base = slot_base(s, t0);
  for (int ci = 0; ci < n_chunks; ++ci) {
    const int tc0 = t0 + ci * C, n = min(C, t1 - tc0);
    const size_t wsi = (size_t)(base + ci) * p.H + h;
    __syncthreads();
    float* gS = p.Sst + wsi * sd;
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      gS[(size_t)d * p.dv + col0 + c] = sS[d * LDT + c];
    }
    state_chunk_loads<DK, T>(p, wsi, tc0, n, h, sW, nullptr, sKh, sg, sr, tid);
    const float* gU = p.Ut + wsi * C * p.dv;
    for (int e = tid; e < C * NS; e += THREADS) {
      const int i = e / NS, c = e % NS;
      sX[i * LDT + c] = gU[(size_t)i * p.dv + col0 + c];
    }
    __syncthreads();
    {
      // X = U~ - W S  [C][NS]
      const int r0 = (tid >> 4) * 4, c0 = (tid & 15) * 2;
      float acc[4][2];
      zero(acc);
      gemm<4, 2, DK>(acc, [&](int i, int k) { return sW[(r0 + i) * LDK + k]; },
                     [&](int k, int j) { return sS[k * LDT + c0 + j]; });
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) sX[(r0 + i) * LDT + c0 + j] -= acc[i][j];
    }
    __syncthreads();
    {
      // S = gamma_C S + Kh^T X  [DK][NS]
      const int r0 = (tid >> 4) * TM, c0 = (tid & 15) * 2;
      float acc[TM][2];
      zero(acc);
      gemm<TM, 2, C>(acc, [&](int i, int k) { return sKh[k * LDK + r0 + i]; },
                     [&](int k, int j) { return sX[k * LDT + c0 + j]; });
      const float gC = expf(sg[C - 1]);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          sS[(r0 + i) * LDT + c0 + j] = fmaf(gC, sS[(r0 + i) * LDT + c0 + j], acc[i][j]);
    }
  }
}

// 3. State gradients, backward: dE_c[:, J] (the gradient at the end of chunk
// c) into the workspace, then dE <- gamma_C dE - W^T (Kh dE) + Qh^T dO[:, J];
// what remains after chunk 0 is grad_S0.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_dstates_kernel(const KParams p) {
  extern __shared__ float smf[];
  using PL = StatePlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TM = DK / 16;
  const int tid = threadIdx.x;
  int s, h, col0;
  state_block(p, s, h, col0);
  int t0, t1;
  seq_range(p, s, t0, t1, false);
  float *sE = smf + PL::S, *sW = smf + PL::W, *sKh = smf + PL::KH, *sQh = smf + PL::QH, *sY = smf + PL::X,
        *sdO = smf + PL::DO;
  float *sg = smf + PL::VEC, *sr = smf + PL::VEC + C;
  const size_t sd = (size_t)DK * p.dv;
  const size_t sb0 = ((size_t)s * p.H + h) * sd;
  for (int e = tid; e < DK * NS; e += THREADS) {
    const int d = e / NS, c = e % NS;
    sE[d * LDT + c] = p.gST ? p.gST[sb0 + (size_t)d * p.dv + col0 + c] : 0.f;
  }
  const int n_chunks = (t1 - t0 + C - 1) / C;
  const long long base = slot_base(s, t0);
  for (int ci = n_chunks - 1; ci >= 0; --ci) {
    const int tc0 = t0 + ci * C, n = min(C, t1 - tc0);
    const size_t wsi = (size_t)(base + ci) * p.H + h;
    __syncthreads();
    float* gE = p.dE + wsi * sd;
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      gE[(size_t)d * p.dv + col0 + c] = sE[d * LDT + c];
    }
    state_chunk_loads<DK, T>(p, wsi, tc0, n, h, sW, sQh, sKh, sg, sr, tid);
    load_rows(sdO, LDT, static_cast<const T*>(p.go), tc0, n, h, p.H, p.dv, col0, NS, tid);
    __syncthreads();
    {
      // Y = Kh dE  [C][NS]
      const int r0 = (tid >> 4) * 4, c0 = (tid & 15) * 2;
      float acc[4][2];
      zero(acc);
      gemm<4, 2, DK>(acc, [&](int i, int k) { return sKh[(r0 + i) * LDK + k]; },
                     [&](int k, int j) { return sE[k * LDT + c0 + j]; });
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) sY[(r0 + i) * LDT + c0 + j] = acc[i][j];
    }
    __syncthreads();
    {
      // dE = gamma_C dE - W^T Y + Qh^T dO  [DK][NS]
      const int r0 = (tid >> 4) * TM, c0 = (tid & 15) * 2;
      float acc[TM][2];
      zero(acc);
      gemm<TM, 2, C>(acc, [&](int i, int k) { return sQh[k * LDK + r0 + i]; },
                     [&](int k, int j) { return sdO[k * LDT + c0 + j]; });
      gemm<TM, 2, C>(acc, [&](int i, int k) { return -sW[k * LDK + r0 + i]; },
                     [&](int k, int j) { return sY[k * LDT + c0 + j]; });
      const float gC = expf(sg[C - 1]);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          sE[(r0 + i) * LDT + c0 + j] = fmaf(gC, sE[(r0 + i) * LDT + c0 + j], acc[i][j]);
    }
  }
  __syncthreads();
  if (p.gS0)
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      p.gS0[sb0 + (size_t)d * p.dv + col0 + c] = sE[d * LDT + c];
    }
}

template <int DK>
struct GradPlan {
  static constexpr int LDK = DK + 1;
  static constexpr int K = 0;
  static constexpr int Q = K + C * LDK;
  static constexpr int KK = Q + C * LDK;
  static constexpr int P = KK + C * LDC;
  static constexpr int T = P + C * LDC;
  static constexpr int S = T + C * LDC;        // [DK][LDT]
  static constexpr int E = S + DK * LDT;       // [DK][LDT]
  static constexpr int TILES = E + DK * LDT;   // 7 x [C][LDT]: V, dO, KS, R, U, dU, dR
  static constexpr int VEC = TILES + 7 * C * LDT;
  static constexpr int FLOATS = VEC + 10 * C + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
  static_assert(7 * C * LDT >= 2 * C * LDC, "dA and dP reuse the tile area");
};

// 4. Per (chunk, head): every gradient of the chunk's tokens.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_grads_kernel(const KParams p) {
  extern __shared__ float smf[];
  using PL = GradPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TN = DK / 16;
  const int tid = threadIdx.x;
  const long long slot = blockIdx.x / p.H;
  const int h = blockIdx.x % p.H;
  int s, c, t0, n;
  if (!slot_chunk(p, slot, s, c, t0, n)) return;
  float *sK = smf + PL::K, *sQ = smf + PL::Q, *sKK = smf + PL::KK, *sP = smf + PL::P, *sT = smf + PL::T;
  float *sS = smf + PL::S, *sE = smf + PL::E;
  float* tiles = smf + PL::TILES;
  float *sV = tiles, *sdO = tiles + C * LDT, *sKS = tiles + 2 * C * LDT, *sR = tiles + 3 * C * LDT,
        *sU = tiles + 4 * C * LDT, *sdU = tiles + 5 * C * LDT, *sdR = tiles + 6 * C * LDT;
  float* vec = smf + PL::VEC;
  Vec V{vec, vec + C, vec + 2 * C, vec + 3 * C, vec + 4 * C};
  float *s_db = vec + 5 * C, *s_dg = vec + 6 * C, *s_kap = vec + 7 * C, *s_red = vec + 8 * C;
  chunk_setup<DK, T>(p, t0, n, h, sK, sQ, sKK, sP, sT, V, vec + 10 * C, tid);

  const size_t wsi = (size_t)slot * p.H + h;
  const size_t sd = (size_t)DK * p.dv;
  const float* gS = p.Sst + wsi * sd;
  const float* gE = p.dE + wsi * sd;
  const int rg = tid >> 4, cg = tid & 15;
  const int r0 = rg * 4;
  // register accumulators (fixed thread -> element map over all tiles)
  float dA[4][4], dP[4][4], dq[4][TN], dk[4][TN];
  zero(dA);
  zero(dP);
  zero(dq);
  zero(dk);
  float rd_db[4] = {0.f, 0.f, 0.f, 0.f}, rd_dg[4] = {0.f, 0.f, 0.f, 0.f}, rd_kap[4] = {0.f, 0.f, 0.f, 0.f};
  float es = 0.f;   // partial <dE, S>
  const T* v = static_cast<const T*>(p.v);
  const T* go = static_cast<const T*>(p.go);

  for (int col0 = 0; col0 < p.dv; col0 += NS) {
    __syncthreads();
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, cc = e % NS;
      const float x = gS[(size_t)d * p.dv + col0 + cc], y = gE[(size_t)d * p.dv + col0 + cc];
      sS[d * LDT + cc] = x;
      sE[d * LDT + cc] = y;
      es = fmaf(x, y, es);
    }
    load_rows(sV, LDT, v, t0, n, h, p.H, p.dv, col0, NS, tid);
    load_rows(sdO, LDT, go, t0, n, h, p.H, p.dv, col0, NS, tid);
    __syncthreads();
    const int c0 = cg * 2;
    {
      // KS = K S_J, KdE = K dE_J; R = diag(b) (V - diag(gamma) KS); dU = diag(r) KdE
      float ks[4][2], ke[4][2];
      zero(ks);
      zero(ke);
#pragma unroll 4
      for (int k = 0; k < DK; ++k) {
        float av[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = sK[(r0 + i) * LDK + k];
        const float b0 = sS[k * LDT + c0], b1 = sS[k * LDT + c0 + 1];
        const float e0 = sE[k * LDT + c0], e1 = sE[k * LDT + c0 + 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ks[i][0] = fmaf(av[i], b0, ks[i][0]);
          ks[i][1] = fmaf(av[i], b1, ks[i][1]);
          ke[i][0] = fmaf(av[i], e0, ke[i][0]);
          ke[i][1] = fmaf(av[i], e1, ke[i][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          sKS[r * LDT + c0 + j] = ks[i][j];
          sR[r * LDT + c0 + j] = V.b[r] * (sV[r * LDT + c0 + j] - V.gam[r] * ks[i][j]);
          sdU[r * LDT + c0 + j] = V.r[r] * ke[i][j];
        }
      }
    }
    __syncthreads();
    {
      // U = T R; kappa partials U_i . (diag(r) KdE)_i
      float acc[4][2];
      zero(acc);
      gemm<4, 2, C>(acc, [&](int i, int k) { return sT[(r0 + i) * LDC + k]; },
                    [&](int k, int j) { return sR[k * LDT + c0 + j]; });
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          sU[(r0 + i) * LDT + c0 + j] = acc[i][j];
          rd_kap[i] = fmaf(acc[i][j], sdU[(r0 + i) * LDT + c0 + j], rd_kap[i]);
        }
    }
    __syncthreads();
    {
      // dU += P^T dO
      float acc[4][2];
      zero(acc);
      gemm<4, 2, C>(acc, [&](int i, int k) { return sP[k * LDC + r0 + i]; },
                    [&](int k, int j) { return sdO[k * LDT + c0 + j]; });
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) sdU[(r0 + i) * LDT + c0 + j] += acc[i][j];
    }
    __syncthreads();
    {
      // dR = T^T dU; grad_v = diag(b) dR; db and dg row partials
      float acc[4][2];
      zero(acc);
      gemm<4, 2, C>(acc, [&](int i, int k) { return sT[k * LDC + r0 + i]; },
                    [&](int k, int j) { return sdU[k * LDT + c0 + j]; });
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float dr = acc[i][j], ksv = sKS[r * LDT + c0 + j];
          sdR[r * LDT + c0 + j] = dr;
          rd_db[i] = fmaf(dr, sV[r * LDT + c0 + j] - V.gam[r] * ksv, rd_db[i]);
          rd_dg[i] = fmaf(-V.b[r] * V.gam[r] * dr, ksv, rd_dg[i]);
        }
        if (r < n) {
          float* gvr = p.gv + ((size_t)(t0 + r) * p.H + h) * p.dv + col0 + c0;
          gvr[0] = V.b[r] * acc[i][0];
          gvr[1] = V.b[r] * acc[i][1];
        }
      }
    }
    __syncthreads();
    {
      // dA += dR U^T, dP += dO U^T  (C x C, K = NS; columns cg + 16 j)
#pragma unroll 4
      for (int k = 0; k < NS; ++k) {
        float ar[4], ao[4], bu[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ar[i] = sdR[(r0 + i) * LDT + k];
          ao[i] = sdO[(r0 + i) * LDT + k];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) bu[j] = sU[(cg + 16 * j) * LDT + k];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dA[i][j] = fmaf(ar[i], bu[j], dA[i][j]);
            dP[i][j] = fmaf(ao[i], bu[j], dP[i][j]);
          }
      }
      // dq += dO S_J^T  (C x DK, K = NS; columns cg + 16 j)
      gemm<4, TN, NS>(dq, [&](int i, int k) { return sdO[(r0 + i) * LDT + k]; },
                      [&](int k, int j) { return sS[(cg + 16 * j) * LDT + k]; });
    }
    __syncthreads();
    // row scalings for dk: dR <- -b gamma dR, U <- r U
    for (int e = tid; e < C * NS; e += THREADS) {
      const int i = e / NS, cc = e % NS;
      sdR[i * LDT + cc] *= -V.b[i] * V.gam[i];
      sU[i * LDT + cc] *= V.r[i];
    }
    __syncthreads();
    {
      // dk += (-b gamma dR) S_J^T + (r U) dE_J^T
      gemm<4, TN, NS>(dk, [&](int i, int k) { return sdR[(r0 + i) * LDT + k]; },
                      [&](int k, int j) { return sS[(cg + 16 * j) * LDT + k]; });
      gemm<4, TN, NS>(dk, [&](int i, int k) { return sU[(r0 + i) * LDT + k]; },
                      [&](int k, int j) { return sE[(cg + 16 * j) * LDT + k]; });
    }
  }

  // ---- row partials -> per-row values (threads with cg == 0 hold the rows)
  {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float qd = 0.f;
#pragma unroll
      for (int j = 0; j < TN; ++j) qd = fmaf(sQ[(r0 + i) * LDK + cg + 16 * j], dq[i][j], qd);
      qd = half_warp_sum(qd);
      const float db = half_warp_sum(rd_db[i]);
      const float dg = half_warp_sum(rd_dg[i]);
      const float kap = half_warp_sum(rd_kap[i]);
      if (cg == 0) {
        const int r = r0 + i;
        s_db[r] = db;
        s_dg[r] = dg + p.scale * V.gam[r] * qd;
        s_kap[r] = kap;
      }
    }
    // <dE, S>
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) es += __shfl_xor_sync(0xffffffffu, es, off);
    if ((tid & 31) == 0) s_red[tid >> 5] = es;
  }
  __syncthreads();
  // dA, dP (unscaled) into the tile area
  float* sdA = tiles;
  float* sdP = tiles + C * LDC;
  {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + i, cc = cg + 16 * j;
        sdA[r * LDC + cc] = (cc < r) ? -dA[i][j] : 0.f;
        sdP[r * LDC + cc] = (cc <= r) ? dP[i][j] : 0.f;
      }
  }
  __syncthreads();
  if (tid < C) {
    // dg and db of row i; then scale dA, dP rows into A' and dP o scale D below
    const int i = tid;
    float dg = s_dg[i] - s_kap[i], db = s_db[i];
    for (int j = 0; j < C; ++j) {
      const float dpij = sdP[i * LDC + j], dpji = sdP[j * LDC + i];
      const float daij = sdA[i * LDC + j], daji = sdA[j * LDC + i];
      dg += dpij * sP[i * LDC + j] - dpji * sP[j * LDC + i];
      dg += daij * V.b[i] * sKK[i * LDC + j] - daji * V.b[j] * sKK[j * LDC + i];
      db = fmaf(daij, sKK[i * LDC + j], db);
    }
    if (i == C - 1) {
      float ksum = 0.f, esum = 0.f;
      for (int j = 0; j < C; ++j) ksum += s_kap[j];
      for (int w = 0; w < THREADS / 32; ++w) esum += s_red[w];
      dg += ksum + V.gam[C - 1] * esum;
    }
    s_dg[i] = dg;
    s_db[i] = db;
  }
  __syncthreads();
  if (tid < 32) {
    // dlog a_m = sum_{i >= m} dg_i (two rows per lane, then a suffix scan)
    const int lane = tid;
    const float x0 = s_dg[2 * lane], x1 = s_dg[2 * lane + 1];
    float suf = x0 + x1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, suf, off);
      if (lane + off < 32) suf += y;
    }
    // suf = sum over pairs lane .. 31
    const float d1 = suf - x0;     // rows 2 lane + 1 .. 63
    const float d0 = suf;          // rows 2 lane .. 63
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int m = 2 * lane + u;
      if (m < n) {
        const size_t ti = (size_t)(t0 + m) * p.H + h;
        p.ga[ti] = (u == 0 ? d0 : d1) / fmaxf(V.a[m], kMinGate);
        p.gb[ti] = s_db[m];
      }
    }
  }
  // A'_ij = dA_ij b_i D_ij, Pb_ij = dP_ij scale D_ij (in place)
  for (int e = tid; e < C * C; e += THREADS) {
    const int i = e / C, j = e % C;
    const float d = (j <= i) ? expf(V.g[i] - V.g[j]) : 0.f;
    sdA[i * LDC + j] *= V.b[i] * d;
    sdP[i * LDC + j] *= p.scale * d;
  }
  __syncthreads();
  {
    // dq = scale diag(gamma) dq + Pb K;  dk += (A' + A'^T) K + Pb^T Q
    float acc[4][TN];
    zero(acc);
    gemm<4, TN, C>(acc, [&](int i, int k) { return sdP[(r0 + i) * LDC + k]; },
                   [&](int k, int j) { return sK[k * LDK + cg + 16 * j]; });
    gemm<4, TN, C>(dk, [&](int i, int k) { return sdA[(r0 + i) * LDC + k] + sdA[k * LDC + r0 + i]; },
                   [&](int k, int j) { return sK[k * LDK + cg + 16 * j]; });
    gemm<4, TN, C>(dk, [&](int i, int k) { return sdP[k * LDC + r0 + i]; },
                   [&](int k, int j) { return sQ[k * LDK + cg + 16 * j]; });
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = r0 + i;
      if (r < n) {
        const size_t row = ((size_t)(t0 + r) * p.H + h) * DK + cg;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          p.gq[row + 16 * j] = fmaf(p.scale * V.gam[r], dq[i][j], acc[i][j]);
          p.gk[row + 16 * j] = dk[i][j];
        }
      }
    }
  }
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static long long n_slots(const gdn_bwd_params* p) {
  return (long long)p->total_tokens / C + 2LL * p->n_seq + 1;
}

template <int DK, typename T>
static gdn_status launch_all(const KParams& kp, const gdn_bwd_params* p, cudaStream_t stream) {
  static std::atomic<bool> set_prep[kMaxDevices], set_st[kMaxDevices], set_dst[kMaxDevices],
      set_gr[kMaxDevices];
  if (smem_attr_once(set_prep, gdn_bwd_prep_kernel<DK, T>, PrepPlan<DK>::BYTES) != cudaSuccess ||
      smem_attr_once(set_st, gdn_bwd_states_kernel<DK, T>, StatePlan<DK>::BYTES) != cudaSuccess ||
      smem_attr_once(set_dst, gdn_bwd_dstates_kernel<DK, T>, StatePlan<DK>::BYTES) != cudaSuccess ||
      smem_attr_once(set_gr, gdn_bwd_grads_kernel<DK, T>, GradPlan<DK>::BYTES) != cudaSuccess)
    return GDN_ERR_CUDA;
  const long long chunk_blocks = kp.n_slots * p->H;
  const long long chain_blocks = (long long)p->n_seq * p->H * (p->dv / NS);
  if (chunk_blocks > 0x7fffffffLL || chain_blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  gdn_bwd_prep_kernel<DK, T><<<(unsigned)chunk_blocks, THREADS, PrepPlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_states_kernel<DK, T><<<(unsigned)chain_blocks, THREADS, StatePlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_dstates_kernel<DK, T><<<(unsigned)chain_blocks, THREADS, StatePlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_grads_kernel<DK, T><<<(unsigned)chunk_blocks, THREADS, GradPlan<DK>::BYTES, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace cbwd

// Workspace of the chunkwise path: W, Qh [slots][H][C][dk], U~ [slots][H][C][dv],
// g [slots][H][C], start states and end-state gradients [slots][H][dk][dv].
size_t bwd_chunk_workspace(const gdn_bwd_params* p) {
  const size_t sh = (size_t)cbwd::n_slots(p) * p->H;
  const size_t C = cbwd::C;
  return cbwd::align256(sh * C * p->dk * 4) * 2 + cbwd::align256(sh * C * p->dv * 4) +
         cbwd::align256(sh * C * 4) + cbwd::align256(sh * (size_t)p->dk * p->dv * 4) * 2;
}

gdn_status launch_bwd_chunk(const gdn_bwd_params* p, unsigned* status, void* ws, cudaStream_t stream) {
  if ((long long)p->n_seq * p->H <= 0) return GDN_OK;
  cbwd::KParams kp;
  kp.q = p->q;
  kp.k = p->k;
  kp.v = p->v;
  kp.go = p->grad_o;
  kp.a = p->a;
  kp.b = p->b;
  kp.S0 = p->S0;
  kp.gST = p->grad_S_T;
  kp.gq = p->grad_q;
  kp.gk = p->grad_k;
  kp.gv = p->grad_v;
  kp.ga = p->grad_a;
  kp.gb = p->grad_b;
  kp.gS0 = p->grad_S0;
  kp.cu = p->cu_seqlens;
  kp.n_seq = p->n_seq;
  kp.seq_len = p->seq_len;
  kp.total = p->total_tokens;
  kp.H = p->H;
  kp.dv = p->dv;
  kp.scale = p->scale;
  kp.n_slots = cbwd::n_slots(p);
  kp.status = status;
  const size_t sh = (size_t)kp.n_slots * p->H;
  const size_t C = cbwd::C;
  char* w = static_cast<char*>(ws);
  kp.W = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * p->dk * 4);
  kp.Qh = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * p->dk * 4);
  kp.Ut = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * p->dv * 4);
  kp.G = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * 4);
  kp.Sst = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * (size_t)p->dk * p->dv * 4);
  kp.dE = reinterpret_cast<float*>(w);
  const bool bf = p->io_dtype == GDN_BF16;
  if (p->dk == 128)
    return bf ? cbwd::launch_all<128, __nv_bfloat16>(kp, p, stream) : cbwd::launch_all<128, float>(kp, p, stream);
  return bf ? cbwd::launch_all<64, __nv_bfloat16>(kp, p, stream) : cbwd::launch_all<64, float>(kp, p, stream);
}

}  // namespace gdn
