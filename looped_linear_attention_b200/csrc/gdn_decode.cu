// One decode step of the gated delta rule for many independent state slots
// (one slot = one sequence x layer x loop state of a looped GDN model; the
// linear-time mixer keeps a fixed-size state, so each step costs the same,
// "LT2: Linear-Time Looped Transformers", §2).
//
// With the state Sigma in R^{dk x dv} (dv contiguous in memory):
//     x_k = Sigma^T k,  x_q = Sigma^T q            (reductions over dk)
//     u   = b (v - a x_k)
//     o   = scale (a x_q + (k . q) u)
//     Sigma <- a Sigma + k u^T                     (in place)
// which is Sigma_t = a (I - b k k^T) Sigma_{t-1} + b k v^T, o = scale Sigma_t^T q.
//
// HBM-bound: each head-state is read once and written once, 128-bit accesses
// coalesced along dv, the state held in registers between the read and the
// write.  One CTA of 8 warps handles one (slot, head, dv block of 32*VEC
// columns); lane l owns VEC consecutive columns and warp w owns DK/8 rows, the
// dk reductions go through shared memory.
#include "common.cuh"

namespace gdn {

__device__ __forceinline__ float4 ld_f4_stream(const float* p) {
  float4 r;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ float2 ld_f2_stream(const float* p) {
  float2 r;
  asm volatile("ld.global.L1::no_allocate.v2.f32 {%0,%1}, [%2];" : "=f"(r.x), "=f"(r.y) : "l"(p));
  return r;
}

template <int DK, int VEC, typename T>
__global__ void __launch_bounds__(256, 2)
    gdn_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ a, const float* __restrict__ b, float* S, T* o,
                      int dv, float scale, unsigned flags) {
  constexpr int RPW = DK / 8;          // rows per warp
  constexpr int COLS = 32 * VEC;       // columns per CTA
  constexpr int KPL = DK / 32;         // q/k elements per lane for the norms
  __shared__ float red[8][2][COLS];

  const int col_blocks = dv / COLS;
  const long long sh = blockIdx.x / col_blocks;   // slot * H + head
  const int cb = blockIdx.x % col_blocks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = cb * COLS + lane * VEC;

  const T* qp = q + sh * DK;
  const T* kp = k + sh * DK;

  // full-vector quantities (every warp computes them; no block sync needed)
  float qq = 0.f, kk = 0.f, kq = 0.f;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const float qe = to_f32(qp[lane + 32 * e]);
    const float ke = to_f32(kp[lane + 32 * e]);
    qq = fmaf(qe, qe, qq);
    kk = fmaf(ke, ke, kk);
    kq = fmaf(ke, qe, kq);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    qq += __shfl_xor_sync(0xffffffffu, qq, off);
    kk += __shfl_xor_sync(0xffffffffu, kk, off);
    kq += __shfl_xor_sync(0xffffffffu, kq, off);
  }
  float nq = 1.f, nk = 1.f;
  if (flags & GDN_QK_L2NORM) {
    nq = 1.0f / sqrtf(qq + kQkNormEps);
    nk = 1.0f / sqrtf(kk + kQkNormEps);
  }
  const float aa = a[sh], bb = b[sh];

  // load this thread's RPW x VEC block of the state
  float s[RPW][VEC];
  float* Sp = S + (sh * DK + warp * RPW) * (long long)dv + c0;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    if constexpr (VEC == 4) {
      const float4 t = ld_f4_stream(Sp + (long long)i * dv);
      s[i][0] = t.x; s[i][1] = t.y; s[i][2] = t.z; s[i][3] = t.w;
    } else {
      const float2 t = ld_f2_stream(Sp + (long long)i * dv);
      s[i][0] = t.x; s[i][1] = t.y;
    }
  }
  float kr[RPW];
  float xk[VEC], xq[VEC];
#pragma unroll
  for (int c = 0; c < VEC; ++c) xk[c] = xq[c] = 0.f;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int r = warp * RPW + i;
    kr[i] = to_f32(kp[r]) * nk;
    const float qr = to_f32(qp[r]) * nq;
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
      xk[c] = fmaf(s[i][c], kr[i], xk[c]);
      xq[c] = fmaf(s[i][c], qr, xq[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < VEC; ++c) {
    red[warp][0][lane * VEC + c] = xk[c];
    red[warp][1][lane * VEC + c] = xq[c];
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < VEC; ++c) {
    float sk = 0.f, sq = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      sk += red[w][0][lane * VEC + c];
      sq += red[w][1][lane * VEC + c];
    }
    xk[c] = sk;
    xq[c] = sq;
  }
  const float kqn = kq * nk * nq;
  const T* vp = v + sh * (long long)dv + c0;
  float u[VEC];
#pragma unroll
  for (int c = 0; c < VEC; ++c) u[c] = bb * (to_f32(vp[c]) - aa * xk[c]);
  if (warp == 0) {
    T* op = o + sh * (long long)dv + c0;
#pragma unroll
    for (int c = 0; c < VEC; ++c) op[c] = from_f32<T>(scale * fmaf(aa, xq[c], kqn * u[c]));
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    float* dst = Sp + (long long)i * dv;
    if constexpr (VEC == 4) {
      float4 t;
      t.x = fmaf(aa, s[i][0], kr[i] * u[0]);
      t.y = fmaf(aa, s[i][1], kr[i] * u[1]);
      t.z = fmaf(aa, s[i][2], kr[i] * u[2]);
      t.w = fmaf(aa, s[i][3], kr[i] * u[3]);
      __stcs(reinterpret_cast<float4*>(dst), t);
    } else {
      float2 t;
      t.x = fmaf(aa, s[i][0], kr[i] * u[0]);
      t.y = fmaf(aa, s[i][1], kr[i] * u[1]);
      __stcs(reinterpret_cast<float2*>(dst), t);
    }
  }
}

template <int DK, typename T>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* a,
                                   const float* b, float* S, void* o, long long NH, int dv,
                                   float scale, unsigned flags, cudaStream_t stream) {
  const bool wide = (dv % 128) == 0;
  const int cols = wide ? 128 : 64;
  const long long blocks = NH * (dv / cols);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (wide)
    gdn_decode_kernel<DK, 4, T><<<(unsigned)blocks, 256, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, a, b, S, (T*)o, dv, scale, flags);
  else
    gdn_decode_kernel<DK, 2, T><<<(unsigned)blocks, 256, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, a, b, S, (T*)o, dv, scale, flags);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* a,
                          const float* b, float* S, void* o, int N, int H, int dk, int dv,
                          gdn_dtype dt, float scale, unsigned flags, cudaStream_t stream) {
  const long long NH = (long long)N * H;
  if (dt == GDN_BF16) {
    return dk == 128 ? launch_decode_t<128, __nv_bfloat16>(q, k, v, a, b, S, o, NH, dv, scale, flags, stream)
                     : launch_decode_t<64, __nv_bfloat16>(q, k, v, a, b, S, o, NH, dv, scale, flags, stream);
  }
  return dk == 128 ? launch_decode_t<128, float>(q, k, v, a, b, S, o, NH, dv, scale, flags, stream)
                   : launch_decode_t<64, float>(q, k, v, a, b, S, o, NH, dv, scale, flags, stream);
}

}  // namespace gdn
