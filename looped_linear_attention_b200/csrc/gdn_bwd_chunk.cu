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
//   1. gdn_bwd_prep_kernel    one CTA per (chunk, head): T, W, U~, Qh, g, and
//                             the state passes' operands in their shared-memory
//                             layouts (W^T, diag(r) K and its transpose)
//   2. gdn_bwd_states_kernel  one CTA per (sequence, head, 32 columns of dv):
//                             the chunk start states S_c, forward in order
//   3. gdn_bwd_dstates_kernel the same grid: dE_c backwards, and grad_S0
//      (both stream each chunk's operands with cp.async into single buffers,
//      each load issued as soon as the product before it has read the buffer)
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
constexpr int LDC = C + 4;        // row stride of C x C tiles (a multiple of 4, = 4 mod 32)
constexpr int LDN = NS + 4;       // row stride of [C][NS] tiles (the same two properties)
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
  float *Wt, *Kh, *Kht;             // per (slot, head): W^T [dk][C], diag(r) K [C][dk], its transpose
  float *Sst, *dE;                  // per (slot, head): [dk][dv]
  unsigned* status;
};

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
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

// Rows [0, n) of a [tokens][H][width] input into shared memory ([C][ld]
// fp32, columns [0, cols)), zeros below: 4 elements per load and per float4
// store (ld, width and cols multiples of 4).
__device__ __forceinline__ float4 ld4(const float* p, size_t i) {
  return __ldg(reinterpret_cast<const float4*>(p + i));
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p, size_t i) {
  const uint2 u = *reinterpret_cast<const uint2*>(p + i);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}
__device__ __forceinline__ void cp_async16(float* smem, const float* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// 16 bytes, or zeros when !take (nothing is read then)
__device__ __forceinline__ void cp_async16z(float* smem, const void* gmem, bool take) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(take ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}
__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float f4(const float4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}

// Shared setup of the prep and grads kernels: K and Q rows (stride DK + 4),
// gate vectors, KK = D o K K^T (strictly lower), P = scale D o Q K^T (lower,
// diagonal included) and T.
template <int DK, typename T>
__device__ __forceinline__ void chunk_setup(const KParams& p, int t0, int n, int h, float* sK, float* sQ,
                                            float* sKK, float* sP, float* sT, Vec V, float* s_carry,
                                            int tid) {
  constexpr int LDK = DK + 4;
  // K and Q rows staged with 16-byte cp.async, every piece in flight (rows
  // past the end read nothing: zero fill): fp32 rows straight into their
  // rows, bf16 rows into the KK and P areas (written only later), then widened
  constexpr bool kF32 = sizeof(T) == 4;
  {
    constexpr int PIECES = DK * (int)sizeof(T) / 16;
    constexpr int RAW = kF32 ? LDK : DK / 2;      // floats per staged row
    float* rk = kF32 ? sK : sKK;
    float* rq = kF32 ? sQ : sP;
    const T* kg = static_cast<const T*>(p.k);
    const T* qg = static_cast<const T*>(p.q);
    for (int e = tid; e < C * PIECES; e += THREADS) {
      const int i = e / PIECES, c = e % PIECES;
      const size_t off = ((size_t)(t0 + min(i, n - 1)) * p.H + h) * DK;
      cp_async16z(rk + i * RAW + 4 * c, reinterpret_cast<const char*>(kg + off) + 16 * c, i < n);
      cp_async16z(rq + i * RAW + 4 * c, reinterpret_cast<const char*>(qg + off) + 16 * c, i < n);
    }
    cp_async_commit();
  }
  chunk_gates(p, t0, n, h, V, s_carry, tid);
  cp_async_wait<0>();
  __syncthreads();
  if constexpr (!kF32) {
    for (int e = tid; e < C * DK / 4; e += THREADS) {
      const int i = e / (DK / 4), c = 4 * (e % (DK / 4));
      const uint2 uk = *reinterpret_cast<const uint2*>(sKK + i * (DK / 2) + c / 2);
      const uint2 uq = *reinterpret_cast<const uint2*>(sP + i * (DK / 2) + c / 2);
      *reinterpret_cast<float4*>(sK + i * LDK + c) = make_float4(bf16_lo(uk.x), bf16_hi(uk.x), bf16_lo(uk.y), bf16_hi(uk.y));
      *reinterpret_cast<float4*>(sQ + i * LDK + c) = make_float4(bf16_lo(uq.x), bf16_hi(uq.x), bf16_lo(uq.y), bf16_hi(uq.y));
    }
    __syncthreads();
  }
  {
    // thread: rows r0 .. r0+3, columns cg + 16 j; both products read K and Q
    // along k four at a time (the row stride DK + 4 keeps the eight rows of a
    // quarter-warp's column reads in distinct banks)
    const int r0 = (tid >> 4) * 4, cg = tid & 15;
    float kk[4][4], qk[4][4];
    zero(kk);
    zero(qk);
#pragma unroll 2
    for (int k = 0; k < DK; k += 4) {
      float4 ak[4], aq[4], bk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ak[i] = *reinterpret_cast<const float4*>(sK + (r0 + i) * LDK + k);
        aq[i] = *reinterpret_cast<const float4*>(sQ + (r0 + i) * LDK + k);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) bk[j] = *reinterpret_cast<const float4*>(sK + (cg + 16 * j) * LDK + k);
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
  static constexpr int LDK = DK + 4;
  static constexpr int K = 0;                 // [C][LDK]
  static constexpr int Q = K + C * LDK;       // [C][LDK]
  static constexpr int W = Q + C * LDK;       // [C][LDK]
  static constexpr int KK = W + C * LDK;      // [C][LDC], then T^T
  static constexpr int P = KK + C * LDC;      // [C][LDC]
  static constexpr int T = P + C * LDC;       // [C][LDC]
  static constexpr int PT = T + C * LDC;      // [C][LDC] P^T
  static constexpr int V = PT + C * LDC;      // [C][LDN]
  static constexpr int VEC = V + C * LDN;     // 5 x C + carry
  static constexpr int FLOATS = VEC + 5 * C + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
  static_assert(BYTES <= 232448, "shared memory of one CTA");
};

// 1. Per (chunk, head): W = T diag(b gamma) K, U~ = T diag(b) V, Qh = scale
// diag(gamma) Q - P W and g, into the workspace.  The products read k-major
// float4 operands: T^T (over KK, free after the solve) and P^T are transposed
// copies.  Thread map as in the gradient kernel (rows 4 rg .. 4 rg + 3;
// C x DK columns 4 cg .. 4 cg + 3 and 64 + 4 cg ..; tile columns cg, cg + 16).
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_prep_kernel(const KParams p) {
  extern __shared__ __align__(16) float smf[];
  using PL = PrepPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int NV = DK / 64;
  const int tid = threadIdx.x;
  const long long slot = blockIdx.x / p.H;
  const int h = blockIdx.x % p.H;
  int s, c, t0, n;
  if (!slot_chunk(p, slot, s, c, t0, n)) return;
  float *sK = smf + PL::K, *sQ = smf + PL::Q, *sW = smf + PL::W, *sKK = smf + PL::KK, *sP = smf + PL::P,
        *sT = smf + PL::T, *sPt = smf + PL::PT, *sV = smf + PL::V;
  float* sTt = sKK;
  Vec V{smf + PL::VEC, smf + PL::VEC + C, smf + PL::VEC + 2 * C, smf + PL::VEC + 3 * C,
        smf + PL::VEC + 4 * C};
  chunk_setup<DK, T>(p, t0, n, h, sK, sQ, sKK, sP, sT, V, smf + PL::VEC + 5 * C, tid);
  for (int e = tid; e < C * C; e += THREADS) {
    const int i = e / C, j = e % C;
    sTt[j * LDC + i] = sT[i * LDC + j];
    sPt[j * LDC + i] = sP[i * LDC + j];
  }
  const size_t wsi = (size_t)slot * p.H + h;
  const int rg = tid >> 4, cg = tid & 15;
  const int r0 = rg * 4;
  if (tid < C) p.G[wsi * C + tid] = V.g[tid];
  {
    // diag(r) K, row-major and transposed, for the state passes
    float* gKh = p.Kh + wsi * C * DK;
    float* gKht = p.Kht + wsi * C * DK;
    for (int e = tid; e < C * DK / 4; e += THREADS) {
      const int i = (e * 4) / DK, d = (e * 4) % DK;
      float4 x = lds4(sK + i * LDK + d);
      const float ri = V.r[i];
      x.x *= ri; x.y *= ri; x.z *= ri; x.w *= ri;
      *reinterpret_cast<float4*>(gKh + (size_t)i * DK + d) = x;
    }
    for (int e = tid; e < C * DK; e += THREADS) {
      const int d = e / C, i = e % C;
      gKht[(size_t)d * C + i] = V.r[i] * sK[i * LDK + d];
    }
  }
  __syncthreads();
  {
    // W = T diag(b gamma) K  [C][DK]
    float acc[4][4 * NV];
    zero(acc);
#pragma unroll 2
    for (int k = 0; k < C; ++k) {
      const float4 a4 = lds4(sTt + k * LDC + r0);
      const float bgk = V.b[k] * V.gam[k];
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float4 b4 = lds4(sK + k * LDK + 64 * w + 4 * cg);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][4 * w + e] = fmaf(f4(a4, i) * bgk, f4(b4, e), acc[i][4 * w + e]);
      }
    }
    float* gW = p.W + wsi * C * DK;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float4 o = make_float4(acc[i][4 * w], acc[i][4 * w + 1], acc[i][4 * w + 2], acc[i][4 * w + 3]);
        *reinterpret_cast<float4*>(sW + (r0 + i) * LDK + 64 * w + 4 * cg) = o;
        *reinterpret_cast<float4*>(gW + (size_t)(r0 + i) * DK + 64 * w + 4 * cg) = o;
      }
  }
  __syncthreads();
  {
    float* gWt = p.Wt + wsi * C * DK;
    for (int e = tid; e < C * DK; e += THREADS) {
      const int d = e / C, i = e % C;
      gWt[(size_t)d * C + i] = sW[i * LDK + d];
    }
  }
  {
    // Qh = scale diag(gamma) Q - P W  [C][DK]
    float acc[4][4 * NV];
    zero(acc);
#pragma unroll 2
    for (int k = 0; k < C; ++k) {
      const float4 a4 = lds4(sPt + k * LDC + r0);
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float4 b4 = lds4(sW + k * LDK + 64 * w + 4 * cg);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[i][4 * w + e] = fmaf(f4(a4, i), f4(b4, e), acc[i][4 * w + e]);
      }
    }
    float* gQ = p.Qh + wsi * C * DK;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float sg = p.scale * V.gam[r0 + i];
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float4 q4 = lds4(sQ + (r0 + i) * LDK + 64 * w + 4 * cg);
        const float4 o = make_float4(sg * q4.x - acc[i][4 * w], sg * q4.y - acc[i][4 * w + 1],
                                     sg * q4.z - acc[i][4 * w + 2], sg * q4.w - acc[i][4 * w + 3]);
        *reinterpret_cast<float4*>(gQ + (size_t)(r0 + i) * DK + 64 * w + 4 * cg) = o;
      }
    }
  }
  // U~ = T diag(b) V  [C][dv], 32 columns at a time; V's rows (io dtype) are
  // staged with cp.async one block ahead, in two buffers over T (free since
  // its transpose; rows past the end read nothing: zero fill)
  float* gU = p.Ut + wsi * C * p.dv;
  constexpr int VP = NS * (int)sizeof(T) / 16;     // 16-byte pieces per row of a block
  constexpr int VROWF = NS * (int)sizeof(T) / 4;   // floats per staged row
  float* sVraw = sT;
  const T* vg = static_cast<const T*>(p.v);
  auto stage_v = [&](int col0, int buf) {
    for (int e = tid; e < C * VP; e += THREADS) {
      const int i = e / VP, c = e % VP;
      const size_t off = ((size_t)(t0 + min(i, n - 1)) * p.H + h) * p.dv + col0;
      cp_async16z(sVraw + buf * C * VROWF + i * VROWF + 4 * c, reinterpret_cast<const char*>(vg + off) + 16 * c,
                  i < n);
    }
    cp_async_commit();
  };
  stage_v(0, 0);
  for (int col0 = 0, buf = 0; col0 < p.dv; col0 += NS, buf ^= 1) {
    if (col0 + NS < p.dv) stage_v(col0 + NS, buf ^ 1);
    else cp_async_commit();
    cp_async_wait<1>();                            // this block's rows
    __syncthreads();                               // and the last block's product is done with sV
    for (int e = tid; e < C * NS; e += THREADS) {
      const int i = e / NS, cc = e % NS;
      const float* raw = sVraw + buf * C * VROWF + i * VROWF;
      const float x = (sizeof(T) == 4) ? raw[cc] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw)[cc]);
      sV[i * LDN + cc] = V.b[i] * x;
    }
    __syncthreads();
    float acc[4][2];
    zero(acc);
#pragma unroll 4
    for (int k = 0; k < C; ++k) {
      const float4 a4 = lds4(sTt + k * LDC + r0);
      const float b0 = sV[k * LDN + cg], b1 = sV[k * LDN + cg + 16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[i][0] = fmaf(f4(a4, i), b0, acc[i][0]);
        acc[i][1] = fmaf(f4(a4, i), b1, acc[i][1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) gU[(size_t)(r0 + i) * p.dv + col0 + cg + 16 * u] = acc[i][u];
  }
  cp_async_wait<0>();
}

// Shared-memory plans of the state passes, 2 CTAs per SM.  Row strides are
// multiples of 4 (16-byte rows for cp.async and float4 reads; tiles of NS
// columns: NS + 4) so that every operand read of the products is one float4
// (4 rows of a transposed operand) or one float2 (2 columns of a tile).
constexpr int LDX = NS + 4;        // [rows][NS] tiles
constexpr int LDCT = C + 4;        // [DK][C] transposed operands
template <int DK>
struct StatesPlan {
  static constexpr int LDK = DK + 4;
  static constexpr int S = 0;                    // [DK][LDX]  state slice
  static constexpr int WT = S + DK * LDX;        // [DK][LDCT] W^T
  static constexpr int KH = WT + DK * LDCT;      // [C][LDK]   diag(r) K
  static constexpr int X = KH + C * LDK;         // 2 x [C][LDX]: U~ of a chunk, then X, in place
  static constexpr int G = X + 2 * C * LDX;      // [C]
  static constexpr int FLOATS = G + C;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};
template <int DK>
struct DStatesPlan {
  static constexpr int LDK = DK + 4;
  static constexpr int E = 0;                    // [DK][LDX]  gradient slice
  static constexpr int KT = E + DK * LDX;        // [DK][LDCT] (diag(r) K)^T, then Qh [C][LDK]
  static constexpr int KT_FLOATS = (DK * LDCT > C * LDK) ? DK * LDCT : C * LDK;
  static constexpr int W = KT + KT_FLOATS;       // [C][LDK]
  static constexpr int Y = W + C * LDK;          // [C][LDX]
  static constexpr int DO = Y + C * LDX;         // [C][LDX]
  static constexpr int G = DO + C * LDX;         // [C]
  static constexpr int FLOATS = G + C;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

// acc[i][j] += sum_k A[k * LDA + i] B[k * LDB + j] (A and B already offset to
// the thread's rows and columns): TM / 4 float4 and one float2 read per k.
template <int TM, int K, int LDA, int LDB>
__device__ __forceinline__ void gemm_v(float (&acc)[TM][2], const float* A, const float* B) {
  static_assert(TM % 4 == 0 && LDA % 4 == 0 && LDB % 2 == 0, "vector operand layout");
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float av[TM];
#pragma unroll
    for (int q = 0; q < TM / 4; ++q) {
      const float4 a4 = *reinterpret_cast<const float4*>(A + k * LDA + 4 * q);
      av[4 * q] = a4.x;
      av[4 * q + 1] = a4.y;
      av[4 * q + 2] = a4.z;
      av[4 * q + 3] = a4.w;
    }
    const float2 b2 = *reinterpret_cast<const float2*>(B + k * LDB);
#pragma unroll
    for (int i = 0; i < TM; ++i) {
      acc[i][0] = fmaf(av[i], b2.x, acc[i][0]);
      acc[i][1] = fmaf(av[i], b2.y, acc[i][1]);
    }
  }
}

// Asynchronous 16-byte copies global -> shared (per thread, in commit groups).
// rows x cols fp32 (cols a multiple of 4) from global (row stride gld) into
// shared memory (row stride sld), 16 bytes per copy.
__device__ __forceinline__ void cp_rows(float* dst, int sld, const float* src, size_t gld, int rows, int cols,
                                        int tid) {
  const int q = cols / 4;
  for (int e = tid; e < rows * q; e += THREADS) {
    const int i = e / q, c = (e % q) * 4;
    cp_async16(dst + i * sld + c, src + (size_t)i * gld + c);
  }
}

// Chain (sequence, head) and column slice of a state-pass block.
__device__ __forceinline__ void state_block(const KParams& p, int& s, int& h, int& col0) {
  const int n_cs = p.dv / NS;
  col0 = (blockIdx.x % n_cs) * NS;
  const int chain = blockIdx.x / n_cs;
  s = chain / p.H;
  h = chain % p.H;
}

// 2. Chunk start states, forward: S_c[:, J] into the workspace, then
// S <- gamma_C S + (diag(r) K)^T (U~[:, J] - W S).  Loads per chunk: group A
// (g, W^T, U~ slice) issued once the previous chunk's first product has read
// W^T, group B (diag(r) K) once its second product has read it.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 2) gdn_bwd_states_kernel(const KParams p) {
  extern __shared__ __align__(16) float smf[];
  using PL = StatesPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TM = DK / 16;
  const int tid = threadIdx.x;
  int s, h, col0;
  state_block(p, s, h, col0);
  int t0, t1;
  seq_range(p, s, t0, t1, tid == 0 && col0 == 0 && h == 0);
  float *sS = smf + PL::S, *sWt = smf + PL::WT, *sKh = smf + PL::KH, *sg = smf + PL::G;
  const size_t sd = (size_t)DK * p.dv;
  const size_t sb0 = ((size_t)s * p.H + h) * sd;
  for (int e = tid; e < DK * NS; e += THREADS) {
    const int d = e / NS, c = e % NS;
    sS[d * LDX + c] = p.S0 ? p.S0[sb0 + (size_t)d * p.dv + col0 + c] : 0.f;
  }
  const int n_chunks = (t1 - t0 + C - 1) / C;
  const long long base = slot_base(s, t0);
  auto wsi_of = [&](int ci) { return (size_t)(base + ci) * p.H + h; };
  auto issue_a = [&](int ci) {
    const size_t w = wsi_of(ci);
    if (tid < C / 4) cp_async16(sg + 4 * tid, p.G + w * C + 4 * tid);
    cp_rows(sWt, LDCT, p.Wt + w * C * DK, C, DK, C, tid);
    cp_rows(smf + PL::X + (ci & 1) * C * LDX, LDX, p.Ut + w * C * p.dv + col0, p.dv, C, NS, tid);
    cp_async_commit();
  };
  auto issue_b = [&](int ci) {
    cp_rows(sKh, LDK, p.Kh + wsi_of(ci) * C * DK, DK, C, DK, tid);
    cp_async_commit();
  };
  if (n_chunks > 0) {
    issue_a(0);
    issue_b(0);
  }
  const int rg = tid >> 4, c0 = (tid & 15) * 2;
  for (int ci = 0; ci < n_chunks; ++ci) {
    float* sX = smf + PL::X + (ci & 1) * C * LDX;
    cp_async_wait<1>();                            // group A of this chunk (B may still fly)
    __syncthreads();
    float* gS = p.Sst + wsi_of(ci) * sd;
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      gS[(size_t)d * p.dv + col0 + c] = sS[d * LDX + c];
    }
    const float gC = expf(sg[C - 1]);
    {
      // X = U~ - W S  [C][NS]: rows 4 rg .. +3, columns c0, c0 + 1
      float acc[4][2];
      zero(acc);
      gemm_v<4, DK, LDCT, LDX>(acc, sWt + rg * 4, sS + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) sX[(rg * 4 + i) * LDX + c0 + j] -= acc[i][j];
    }
    __syncthreads();                               // W^T and g are free; X complete
    if (ci + 1 < n_chunks) {
      issue_a(ci + 1);
      cp_async_wait<1>();                          // group B of this chunk
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    {
      // S = gamma_C S + Kh^T X  [DK][NS]: rows TM rg .. +TM-1
      float acc[TM][2];
      zero(acc);
      gemm_v<TM, C, LDK, LDX>(acc, sKh + rg * TM, sX + c0);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          sS[(rg * TM + i) * LDX + c0 + j] = fmaf(gC, sS[(rg * TM + i) * LDX + c0 + j], acc[i][j]);
    }
    __syncthreads();                               // diag(r) K is free
    if (ci + 1 < n_chunks) issue_b(ci + 1);
  }
  cp_async_wait<0>();
}

// 3. State gradients, backward: dE_c[:, J] (the gradient at the end of chunk
// c) into the workspace, then dE <- gamma_C dE - W^T (Kh dE) + Qh^T dO[:, J];
// what remains after chunk 0 is grad_S0.  Kh^T and then Qh share one buffer.
// Loads per chunk c: Qh once Kh dE has read Kh^T; W and g of chunk c - 1 once
// W^T Y has read W; Kh^T of chunk c - 1 once Qh^T dO has read Qh; dO of chunk
// c - 1 through registers, requested at the top of chunk c.
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 2) gdn_bwd_dstates_kernel(const KParams p) {
  extern __shared__ __align__(16) float smf[];
  using PL = DStatesPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int TM = DK / 16;
  constexpr int DO_PER_THREAD = C * NS / THREADS;
  const int tid = threadIdx.x;
  int s, h, col0;
  state_block(p, s, h, col0);
  int t0, t1;
  seq_range(p, s, t0, t1, false);
  float *sE = smf + PL::E, *sKt = smf + PL::KT, *sW = smf + PL::W, *sY = smf + PL::Y, *sdO = smf + PL::DO;
  float *sQh = sKt, *sg = smf + PL::G;
  const size_t sd = (size_t)DK * p.dv;
  const size_t sb0 = ((size_t)s * p.H + h) * sd;
  for (int e = tid; e < DK * NS; e += THREADS) {
    const int d = e / NS, c = e % NS;
    sE[d * LDX + c] = p.gST ? p.gST[sb0 + (size_t)d * p.dv + col0 + c] : 0.f;
  }
  const int n_chunks = (t1 - t0 + C - 1) / C;
  const long long base = slot_base(s, t0);
  const T* go = static_cast<const T*>(p.go);
  auto wsi_of = [&](int ci) { return (size_t)(base + ci) * p.H + h; };
  auto issue_w = [&](int ci) {                     // W and g of chunk ci
    const size_t w = wsi_of(ci);
    if (tid < C / 4) cp_async16(sg + 4 * tid, p.G + w * C + 4 * tid);
    cp_rows(sW, LDK, p.W + w * C * DK, DK, C, DK, tid);
    cp_async_commit();
  };
  auto issue_kt = [&](int ci) {                    // (diag(r) K)^T of chunk ci
    cp_rows(sKt, LDCT, p.Kht + wsi_of(ci) * C * DK, C, DK, C, tid);
    cp_async_commit();
  };
  T dor[DO_PER_THREAD];                            // dO of the next chunk, in flight (raw)
  bool dov[DO_PER_THREAD];
  auto load_do = [&](int ci) {
    const int tc0 = t0 + ci * C, n = min(C, t1 - tc0);
#pragma unroll
    for (int u = 0; u < DO_PER_THREAD; ++u) {
      const int e = tid + THREADS * u, i = e / NS, c = e % NS;
      dov[u] = i < n;
      if (dov[u]) dor[u] = go[((size_t)(tc0 + i) * p.H + h) * p.dv + col0 + c];
    }
  };
  auto store_do = [&]() {
#pragma unroll
    for (int u = 0; u < DO_PER_THREAD; ++u) {
      const int e = tid + THREADS * u, i = e / NS, c = e % NS;
      sdO[i * LDX + c] = dov[u] ? to_float(dor[u]) : 0.f;
    }
  };
  if (n_chunks > 0) {
    issue_w(n_chunks - 1);
    issue_kt(n_chunks - 1);
    load_do(n_chunks - 1);
    store_do();
  }
  const int rg = tid >> 4, c0 = (tid & 15) * 2;
  for (int ci = n_chunks - 1; ci >= 0; --ci) {
    cp_async_wait<0>();                            // W, g and Kh^T of this chunk
    __syncthreads();
    float* gE = p.dE + wsi_of(ci) * sd;
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      gE[(size_t)d * p.dv + col0 + c] = sE[d * LDX + c];
    }
    if (ci > 0) load_do(ci - 1);                   // registers; stored after this chunk's dO is read
    const float gC = expf(sg[C - 1]);
    {
      // Y = Kh dE  [C][NS]
      float acc[4][2];
      zero(acc);
      gemm_v<4, DK, LDCT, LDX>(acc, sKt + rg * 4, sE + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) sY[(rg * 4 + i) * LDX + c0 + j] = acc[i][j];
    }
    __syncthreads();                               // Kh^T is free; Y complete
    cp_rows(sQh, LDK, p.Qh + wsi_of(ci) * C * DK, DK, C, DK, tid);
    cp_async_commit();
    float accW[TM][2];
    zero(accW);
    gemm_v<TM, C, LDK, LDX>(accW, sW + rg * TM, sY + c0);
    __syncthreads();                               // W and g are free
    if (ci > 0) {
      issue_w(ci - 1);
      cp_async_wait<1>();                          // Qh of this chunk
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    {
      // dE = gamma_C dE - W^T Y + Qh^T dO  [DK][NS]
      float accQ[TM][2];
      zero(accQ);
      gemm_v<TM, C, LDK, LDX>(accQ, sQh + rg * TM, sdO + c0);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
          sE[(rg * TM + i) * LDX + c0 + j] =
              fmaf(gC, sE[(rg * TM + i) * LDX + c0 + j], accQ[i][j] - accW[i][j]);
    }
    __syncthreads();                               // Qh and dO are free
    if (ci > 0) {
      issue_kt(ci - 1);
      store_do();
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (p.gS0)
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, c = e % NS;
      p.gS0[sb0 + (size_t)d * p.dv + col0 + c] = sE[d * LDX + c];
    }
}

// Shared memory of the gradient kernel.  Every product reads float4 operands
// in one of two patterns: "rows along k" (A[i][k..k+3] and B[j][k..k+3], both
// row-major along the contraction) or "k-major" (A[k][i..i+3] and
// B[k][j..j+3]); each small matrix is kept in the layout its products need,
// some in both (dO, dR and U as [C][NS] rows and as [NS][C] transposes).
// Row strides are multiples of 4 and = 4 mod 32 (conflict-free float4 reads
// of the 8 rows a quarter-warp touches).
template <int DK>
struct GradPlan {
  static constexpr int LDK = DK + 4;
  static constexpr int K = 0;                    // [C][LDK]
  static constexpr int Q = K + C * LDK;          // [C][LDK]
  static constexpr int KK = Q + C * LDK;         // [C][LDC] D o K K^T, strictly lower
  static constexpr int P = KK + C * LDC;         // [C][LDC] scale D o Q K^T, lower
  static constexpr int T = P + C * LDC;          // [C][LDC]
  static constexpr int ST = T + C * LDC;         // [NS][LDK] S_J^T (tile of the start state)
  static constexpr int ET = ST + NS * LDK;       // [NS][LDK] dE_J^T
  static constexpr int TILES = ET + NS * LDK;
  // tiles: dO, U, dU (then dR) as [C][LDN]; R^T, dO^T, (r U)^T, (-b gamma dR)^T as [NS][LDC]
  static constexpr int DO = TILES;
  static constexpr int U = DO + C * LDN;
  static constexpr int DU = U + C * LDN;
  static constexpr int RT = DU + C * LDN;
  static constexpr int DOT = RT + NS * LDC;
  static constexpr int UT = DOT + NS * LDC;
  static constexpr int DRT = UT + NS * LDC;
  static constexpr int VEC = DRT + NS * LDC;
  static constexpr int FLOATS = VEC + 10 * C + 4;
  static constexpr size_t BYTES = (size_t)FLOATS * 4;
  static_assert(VEC - TILES >= 3 * C * LDC, "the final phase's three C x C matrices reuse the tile area");
  static_assert(DU - U + C * LDN >= DK * NS && DRT - UT + NS * LDC >= DK * NS,
                "a column block's S and dE rows are staged over U / dU and U^T / dR^T");
  static_assert(BYTES <= 232448, "shared memory of one CTA");
};


// 4. Per (chunk, head): every gradient of the chunk's tokens.  Thread maps
// (rg = tid / 16, cg = tid % 16; rows 4 rg .. 4 rg + 3 everywhere):
//   [C][NS] tiles: columns cg, cg + 16 (two per thread);
//   C x C:         columns cg + 16 j, j < 4;
//   C x DK:        columns 4 cg .. 4 cg + 3 (and 64 + 4 cg .. for DK = 128).
template <int DK, typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_grads_kernel(const KParams p) {
  extern __shared__ __align__(16) float smf[];
  using PL = GradPlan<DK>;
  constexpr int LDK = PL::LDK;
  constexpr int NV = DK / 64;                    // float4 column groups per thread in C x DK
  const int tid = threadIdx.x;
  const long long slot = blockIdx.x / p.H;
  const int h = blockIdx.x % p.H;
  int s, c, t0, n;
  if (!slot_chunk(p, slot, s, c, t0, n)) return;
  float *sK = smf + PL::K, *sQ = smf + PL::Q, *sKK = smf + PL::KK, *sP = smf + PL::P, *sT = smf + PL::T;
  float *sSt = smf + PL::ST, *sEt = smf + PL::ET;
  float *sdO = smf + PL::DO, *sU = smf + PL::U, *sdU = smf + PL::DU, *sRt = smf + PL::RT,
        *sdOt = smf + PL::DOT, *sUt = smf + PL::UT, *sdRt = smf + PL::DRT;
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
  // register accumulators (the same thread -> element map over all tiles)
  float dA[4][4], dP[4][4], dq[4][4 * NV], dk[4][4 * NV];
  zero(dA);
  zero(dP);
  zero(dq);
  zero(dk);
  float rd_db[4] = {0.f, 0.f, 0.f, 0.f}, rd_dg[4] = {0.f, 0.f, 0.f, 0.f}, rd_kap[4] = {0.f, 0.f, 0.f, 0.f};
  float es = 0.f;   // partial <dE, S>
  float gam[4], bb[4], rr[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    gam[i] = V.gam[r0 + i];
    bb[i] = V.b[r0 + i];
    rr[i] = V.r[r0 + i];
  }
  const T* v = static_cast<const T*>(p.v);
  const T* go = static_cast<const T*>(p.go);

  for (int col0 = 0; col0 < p.dv; col0 += NS) {
    __syncthreads();
    // tiles of S and dE: [DK][NS] rows by 16-byte cp.async into the U / dU
    // and U^T / dR^T areas (this block writes them only after its first
    // product), transposed below into [NS][DK]; dO (rows and transpose); V
    // (registers)
    float* stS = sU;                               // U and dU are adjacent: DK x NS floats fit
    float* stE = sUt;                              // so are U^T and dR^T
    for (int e = tid; e < DK * NS / 4; e += THREADS) {
      const int d = e / (NS / 4), c4 = 4 * (e % (NS / 4));
      cp_async16(stS + d * NS + c4, gS + (size_t)d * p.dv + col0 + c4);
      cp_async16(stE + d * NS + c4, gE + (size_t)d * p.dv + col0 + c4);
    }
    // dO rows of the block (io dtype) staged over R^T, which this block
    // writes only after the next barrier (rows past the end: zero fill)
    constexpr int OP = NS * (int)sizeof(T) / 16;
    constexpr int OROW = NS * (int)sizeof(T) / 4;
    for (int e = tid; e < C * OP; e += THREADS) {
      const int i = e / OP, c = e % OP;
      const size_t off = ((size_t)(t0 + min(i, n - 1)) * p.H + h) * p.dv + col0;
      cp_async16z(sRt + i * OROW + 4 * c, reinterpret_cast<const char*>(go + off) + 16 * c, i < n);
    }
    cp_async_commit();
    float vv[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        vv[i][u] = (r0 + i < n) ? ldx(v, ((size_t)(t0 + r0 + i) * p.H + h) * p.dv + col0 + cg + 16 * u) : 0.f;
    cp_async_wait<0>();
    __syncthreads();
    // S and dE transposed; the partial <dE, S> over this thread's elements
    for (int e = tid; e < DK * NS; e += THREADS) {
      const int d = e / NS, cc = e % NS;
      const float x = stS[e], y = stE[e];
      sSt[cc * LDK + d] = x;
      sEt[cc * LDK + d] = y;
      es = fmaf(x, y, es);
    }
    // dO into rows and transpose
    for (int e = tid; e < C * NS; e += THREADS) {
      const int i = e / NS, cc = e % NS;
      const float* raw = sRt + i * OROW;
      const float x = (sizeof(T) == 4) ? raw[cc] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw)[cc]);
      sdO[i * LDN + cc] = x;
      sdOt[cc * LDC + i] = x;
    }
    __syncthreads();
    // KS = K S_J, KdE = K dE_J (rows along k); R = diag(b) (V - diag(gamma) KS) -> R^T;
    // the first part of dU, diag(r) KdE, stays in registers
    float ks[4][2], du0[4][2];
    {
      float ke[4][2];
      zero(ks);
      zero(ke);
#pragma unroll 2
      for (int k = 0; k < DK; k += 4) {
        float4 a[4], bs[2], be[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = lds4(sK + (r0 + i) * LDK + k);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          bs[u] = lds4(sSt + (cg + 16 * u) * LDK + k);
          be[u] = lds4(sEt + (cg + 16 * u) * LDK + k);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            ks[i][u] = dot4(a[i], bs[u], ks[i][u]);
            ke[i][u] = dot4(a[i], be[u], ke[i][u]);
          }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          sRt[(cg + 16 * u) * LDC + r0 + i] = bb[i] * (vv[i][u] - gam[i] * ks[i][u]);
          du0[i][u] = rr[i] * ke[i][u];
        }
    }
    __syncthreads();
    {
      // U = T R (rows along k), into U rows and (r U)^T; kappa partials.
      // dU = diag(r) KdE + P^T dO (k-major), into dU rows.
      float uu[4][2], pd[4][2];
      zero(uu);
      zero(pd);
#pragma unroll 2
      for (int k = 0; k < C; k += 4) {
        float4 a[4], b[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = lds4(sT + (r0 + i) * LDC + k);
#pragma unroll
        for (int u = 0; u < 2; ++u) b[u] = lds4(sRt + (cg + 16 * u) * LDC + k);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int u = 0; u < 2; ++u) uu[i][u] = dot4(a[i], b[u], uu[i][u]);
      }
#pragma unroll 4
      for (int k = 0; k < C; ++k) {
        const float4 a4 = lds4(sP + k * LDC + r0);
        const float b0 = sdO[k * LDN + cg], b1 = sdO[k * LDN + cg + 16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pd[i][0] = fmaf(f4(a4, i), b0, pd[i][0]);
          pd[i][1] = fmaf(f4(a4, i), b1, pd[i][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = cg + 16 * u;
          sU[(r0 + i) * LDN + cc] = uu[i][u];
          sUt[cc * LDC + r0 + i] = rr[i] * uu[i][u];
          rd_kap[i] = fmaf(uu[i][u], du0[i][u], rd_kap[i]);
          sdU[(r0 + i) * LDN + cc] = du0[i][u] + pd[i][u];
        }
    }
    __syncthreads();
    float dr[4][2];
    {
      // dR = T^T dU (k-major); grad_v = diag(b) dR; db and dg row partials
      zero(dr);
#pragma unroll 4
      for (int k = 0; k < C; ++k) {
        const float4 a4 = lds4(sT + k * LDC + r0);
        const float b0 = sdU[k * LDN + cg], b1 = sdU[k * LDN + cg + 16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dr[i][0] = fmaf(f4(a4, i), b0, dr[i][0]);
          dr[i][1] = fmaf(f4(a4, i), b1, dr[i][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          rd_db[i] = fmaf(dr[i][u], vv[i][u] - gam[i] * ks[i][u], rd_db[i]);
          rd_dg[i] = fmaf(-bb[i] * gam[i] * dr[i][u], ks[i][u], rd_dg[i]);
          if (r < n) p.gv[((size_t)(t0 + r) * p.H + h) * p.dv + col0 + cg + 16 * u] = bb[i] * dr[i][u];
        }
      }
    }
    __syncthreads();                               // every read of dU is done: dR replaces it
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int cc = cg + 16 * u;
        sdU[(r0 + i) * LDN + cc] = dr[i][u];
        sdRt[cc * LDC + r0 + i] = -bb[i] * gam[i] * dr[i][u];
      }
    __syncthreads();
    {
      // dA += dR U^T, dP += dO U^T (rows along k)
#pragma unroll 2
      for (int k = 0; k < NS; k += 4) {
        float4 ar[4], ao[4], bu[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ar[i] = lds4(sdU + (r0 + i) * LDN + k);
          ao[i] = lds4(sdO + (r0 + i) * LDN + k);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) bu[j] = lds4(sU + (cg + 16 * j) * LDN + k);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dA[i][j] = dot4(ar[i], bu[j], dA[i][j]);
            dP[i][j] = dot4(ao[i], bu[j], dP[i][j]);
          }
      }
      // dq += dO S_J^T; dk += (-b gamma dR) S_J^T + (r U) dE_J^T (k-major)
#pragma unroll 2
      for (int k = 0; k < NS; ++k) {
        const float4 ao = lds4(sdOt + k * LDC + r0), ar = lds4(sdRt + k * LDC + r0), au = lds4(sUt + k * LDC + r0);
#pragma unroll
        for (int w = 0; w < NV; ++w) {
          const float4 bs = lds4(sSt + k * LDK + 64 * w + 4 * cg), be = lds4(sEt + k * LDK + 64 * w + 4 * cg);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              dq[i][4 * w + e] = fmaf(f4(ao, i), f4(bs, e), dq[i][4 * w + e]);
              dk[i][4 * w + e] = fmaf(f4(ar, i), f4(bs, e), fmaf(f4(au, i), f4(be, e), dk[i][4 * w + e]));
            }
        }
      }
    }
  }
  __syncthreads();                                 // the tile area is free

  // ---- row partials -> per-row values (threads with cg == 0 hold the rows)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float qd = 0.f;
#pragma unroll
    for (int w = 0; w < NV; ++w)
#pragma unroll
      for (int e = 0; e < 4; ++e) qd = fmaf(sQ[(r0 + i) * LDK + 64 * w + 4 * cg + e], dq[i][4 * w + e], qd);
    qd = half_warp_sum(qd);
    const float db = half_warp_sum(rd_db[i]);
    const float dg = half_warp_sum(rd_dg[i]);
    const float kap = half_warp_sum(rd_kap[i]);
    if (cg == 0) {
      const int r = r0 + i;
      s_db[r] = db;
      s_dg[r] = dg + p.scale * gam[i] * qd;
      s_kap[r] = kap;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) es += __shfl_xor_sync(0xffffffffu, es, off);
  if ((tid & 31) == 0) s_red[tid >> 5] = es;
  // dA, dP (unscaled) into the tile area
  float* sdA = smf + PL::TILES;
  float* sdP = sdA + C * LDC;
  float* sPbT = sdP + C * LDC;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + i, cc = cg + 16 * j;
      sdA[r * LDC + cc] = (cc < r) ? -dA[i][j] : 0.f;
      sdP[r * LDC + cc] = (cc <= r) ? dP[i][j] : 0.f;
    }
  __syncthreads();
  if (tid < C) {
    // dg and db of row i
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
  // Pb = dP o scale D (also transposed) and M = A' + A'^T, A'_ij = dA_ij b_i D_ij:
  // computed into registers, then written over dA and dP
  {
    float pb[16], mm[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int e = tid + THREADS * m, i = e / C, j = e % C;
      const float dij = (j <= i) ? expf(V.g[i] - V.g[j]) : 0.f;
      const float dji = (i <= j) ? expf(V.g[j] - V.g[i]) : 0.f;
      pb[m] = sdP[i * LDC + j] * p.scale * dij;
      mm[m] = sdA[i * LDC + j] * V.b[i] * dij + sdA[j * LDC + i] * V.b[j] * dji;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int e = tid + THREADS * m, i = e / C, j = e % C;
      sdP[i * LDC + j] = pb[m];
      sPbT[j * LDC + i] = pb[m];
      sdA[i * LDC + j] = mm[m];
    }
  }
  __syncthreads();
  {
    // dq = scale diag(gamma) dq + Pb K;  dk += M K + Pb^T Q  (k-major)
    float acc[4][4 * NV];
    zero(acc);
#pragma unroll 2
    for (int k = 0; k < C; ++k) {
      const float4 apt = lds4(sPbT + k * LDC + r0), am = lds4(sdA + k * LDC + r0), ap = lds4(sdP + k * LDC + r0);
#pragma unroll
      for (int w = 0; w < NV; ++w) {
        const float4 bk = lds4(sK + k * LDK + 64 * w + 4 * cg), bq = lds4(sQ + k * LDK + 64 * w + 4 * cg);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[i][4 * w + e] = fmaf(f4(apt, i), f4(bk, e), acc[i][4 * w + e]);
            dk[i][4 * w + e] = fmaf(f4(am, i), f4(bk, e), fmaf(f4(ap, i), f4(bq, e), dk[i][4 * w + e]));
          }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = r0 + i;
      if (r < n) {
        const size_t row = ((size_t)(t0 + r) * p.H + h) * DK;
#pragma unroll
        for (int w = 0; w < NV; ++w) {
          float4 oq, ok;
          oq.x = fmaf(p.scale * gam[i], dq[i][4 * w + 0], acc[i][4 * w + 0]);
          oq.y = fmaf(p.scale * gam[i], dq[i][4 * w + 1], acc[i][4 * w + 1]);
          oq.z = fmaf(p.scale * gam[i], dq[i][4 * w + 2], acc[i][4 * w + 2]);
          oq.w = fmaf(p.scale * gam[i], dq[i][4 * w + 3], acc[i][4 * w + 3]);
          ok = make_float4(dk[i][4 * w + 0], dk[i][4 * w + 1], dk[i][4 * w + 2], dk[i][4 * w + 3]);
          *reinterpret_cast<float4*>(p.gq + row + 64 * w + 4 * cg) = oq;
          *reinterpret_cast<float4*>(p.gk + row + 64 * w + 4 * cg) = ok;
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
      smem_attr_once(set_st, gdn_bwd_states_kernel<DK, T>, StatesPlan<DK>::BYTES) != cudaSuccess ||
      smem_attr_once(set_dst, gdn_bwd_dstates_kernel<DK, T>, DStatesPlan<DK>::BYTES) != cudaSuccess ||
      smem_attr_once(set_gr, gdn_bwd_grads_kernel<DK, T>, GradPlan<DK>::BYTES) != cudaSuccess)
    return GDN_ERR_CUDA;
  const long long chunk_blocks = kp.n_slots * p->H;
  const long long chain_blocks = (long long)p->n_seq * p->H * (p->dv / NS);
  if (chunk_blocks > 0x7fffffffLL || chain_blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  gdn_bwd_prep_kernel<DK, T><<<(unsigned)chunk_blocks, THREADS, PrepPlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_states_kernel<DK, T><<<(unsigned)chain_blocks, THREADS, StatesPlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_dstates_kernel<DK, T><<<(unsigned)chain_blocks, THREADS, DStatesPlan<DK>::BYTES, stream>>>(kp);
  gdn_bwd_grads_kernel<DK, T><<<(unsigned)chunk_blocks, THREADS, GradPlan<DK>::BYTES, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace cbwd

// Workspace of the chunkwise path: W, Qh, W^T, diag(r) K and its transpose
// [slots][H][C x dk], U~ [slots][H][C][dv], g [slots][H][C], start states and
// end-state gradients [slots][H][dk][dv].
size_t bwd_chunk_workspace(const gdn_bwd_params* p) {
  const size_t sh = (size_t)cbwd::n_slots(p) * p->H;
  const size_t C = cbwd::C;
  return cbwd::align256(sh * C * p->dk * 4) * 5 + cbwd::align256(sh * C * p->dv * 4) +
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
  kp.Wt = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * p->dk * 4);
  kp.Kh = reinterpret_cast<float*>(w);
  w += cbwd::align256(sh * C * p->dk * 4);
  kp.Kht = reinterpret_cast<float*>(w);
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
