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
// HBM-bound: each head-state is read once and written once.  Two kernels:
//   * gdn_decode_stream_kernel (dk = dv = 128, bf16 tokens): persistent, one
//     CTA per SM; states move by bulk asynchronous copies through a 3-stage
//     shared-memory ring, so copies of neighbouring items overlap the math.
//   * gdn_decode_kernel (every other shape): one CTA of 8 warps per (slot,
//     head, dv block of 32*VEC columns), 128-bit accesses coalesced along dv,
//     the state held in registers between the read and the write; lane l owns
//     VEC consecutive columns and warp w owns DK/8 rows.
// In both, the dk reductions go through shared memory.
//
// With GDN_CHANNEL_GATE the decay is per channel (the KDA variant:
// Sigma_t = (I - b k k^T) Diag(a) Sigma_{t-1} + b k v^T, a in (0, 1]^{dk}, read
// from a [slots][H][dk]): then x_k = (Diag(a) Sigma)^T k and x_q likewise,
// u = b (v - x_k), o = scale (x_q + (k . q) u), and row r of the state becomes
// a_r Sigma_r + k_r u^T; with a scalar gate these are the lines above.  Optionally the output
// takes the looped block's epilogue (include/gdn.h, gdn_decode_step_looped):
// the head-wise sigmoid gate, then the loop residual o <- round(o) + rho (.) h_prev.
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

// Output epilogue of the looped block for one output element: the gate factor
// og (1 without a gate), then, with the residual, round to the io dtype and add
// rho (.) h_prev in fp32.
struct Epilogue {
  const float* gate;    // [slots][H] logits, or null
  const void* h_prev;   // [slots][H*dv] io dtype, or null
  const float* rho;     // [H*dv]
  int H;
};
__device__ __forceinline__ float gate_factor(const Epilogue& ep, long long sh) {
  return ep.gate ? 1.f / (1.f + __expf(-__ldg(ep.gate + sh))) : 1.f;
}
template <typename T>
__device__ __forceinline__ T epilogue_out(const Epilogue& ep, float y, long long sh, int dv, int col) {
  if (!ep.h_prev) return from_f32<T>(y);
  const long long h = sh % ep.H;
  const float hp = to_f32(static_cast<const T*>(ep.h_prev)[sh * dv + col]);
  return from_f32<T>(fmaf(__ldg(ep.rho + h * dv + col), hp, to_f32(from_f32<T>(y))));
}

template <int DK, int VEC, typename T, bool CG>
__global__ void __launch_bounds__(256, 2)
    gdn_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ a, const float* __restrict__ b, float* S, T* o,
                      int dv, float scale, unsigned flags, const Epilogue ep) {
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
  const float aa = CG ? 1.f : a[sh], bb = b[sh];

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
  float kr[RPW], ar[RPW];              // key entries and the decay of each row
  float xk[VEC], xq[VEC];
#pragma unroll
  for (int c = 0; c < VEC; ++c) xk[c] = xq[c] = 0.f;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int r = warp * RPW + i;
    kr[i] = to_f32(kp[r]) * nk;
    ar[i] = CG ? __ldg(a + sh * DK + r) : aa;
    const float qr = to_f32(qp[r]) * nq;
    const float kw = CG ? kr[i] * ar[i] : kr[i];
    const float qw = CG ? qr * ar[i] : qr;
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
      xk[c] = fmaf(s[i][c], kw, xk[c]);
      xq[c] = fmaf(s[i][c], qw, xq[c]);
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
    const float og = gate_factor(ep, sh);
#pragma unroll
    for (int c = 0; c < VEC; ++c)
      op[c] = epilogue_out<T>(ep, og * (scale * fmaf(aa, xq[c], kqn * u[c])), sh, dv, c0 + c);
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    float* dst = Sp + (long long)i * dv;
    if constexpr (VEC == 4) {
      float4 t;
      t.x = fmaf(ar[i], s[i][0], kr[i] * u[0]);
      t.y = fmaf(ar[i], s[i][1], kr[i] * u[1]);
      t.z = fmaf(ar[i], s[i][2], kr[i] * u[2]);
      t.w = fmaf(ar[i], s[i][3], kr[i] * u[3]);
      __stcs(reinterpret_cast<float4*>(dst), t);
    } else {
      float2 t;
      t.x = fmaf(ar[i], s[i][0], kr[i] * u[0]);
      t.y = fmaf(ar[i], s[i][1], kr[i] * u[1]);
      __stcs(reinterpret_cast<float2*>(dst), t);
    }
  }
}

// Streaming variant for dk = dv = 128 with bf16 tokens: one persistent CTA per
// SM walks (slot, head) items; each item's 64 KB state and its q, k, v arrive
// by bulk asynchronous copies into a 3-stage shared-memory ring (two items
// ahead), the CTA computes from shared memory and writes the updated state
// back with a bulk store, so loads and stores of neighbouring items overlap
// the arithmetic and every SM keeps about 130 KB in flight.
namespace dec {
constexpr int DK = 128, DV = 128, THREADS = 256, STAGES = 3;
constexpr uint32_t STATE_BYTES = DK * DV * 4;                 // 65536
constexpr uint32_t VEC_BYTES = 128 * 2;                       // one bf16 vector
constexpr uint32_t GATE_VEC_BYTES = DK * 4;                  // per-channel decay (fp32)
// stage: state | q | k | v [| a, with the per-channel gate]
template <bool CG>
struct Ring {
  static constexpr uint32_t STAGE_BYTES = STATE_BYTES + 3 * VEC_BYTES + (CG ? GATE_VEC_BYTES : 0);
  static constexpr uint32_t OFF_RED = STAGES * STAGE_BYTES;   // [8 warps][2][128] fp32 partial sums
  static constexpr uint32_t OFF_BAR = OFF_RED + 8 * 2 * DV * 4;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
  static_assert(SMEM_BYTES <= 232448, "decode ring exceeds shared memory");
  static_assert(STAGE_BYTES % 128 == 0, "stage alignment");
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <bool CG>
__global__ void __launch_bounds__(THREADS, 1)
    gdn_decode_stream_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                             const __nv_bfloat16* __restrict__ v, const float* __restrict__ a,
                             const float* __restrict__ b, float* S, __nv_bfloat16* o, long long NH,
                             float scale, unsigned flags, unsigned* status, const Epilogue ep) {
  using R = Ring<CG>;
  constexpr uint32_t STAGE_BYTES = R::STAGE_BYTES;
  extern __shared__ __align__(128) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + R::OFF_BAR);
  float* red = reinterpret_cast<float*>(dsm + R::OFF_RED);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + R::OFF_BAR + 8 * STAGES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long first = blockIdx.x, step = gridDim.x;
  const int n_items = (first < NH) ? (int)((NH - first + step - 1) / step) : 0;
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // thread 0: item n of this CTA into stage n % STAGES
  auto issue = [&](int n) {
    const long long sh = first + (long long)n * step;
    uint8_t* st = dsm + (n % STAGES) * STAGE_BYTES;
    uint64_t* bar = &full[n % STAGES];
    mbar_arrive_expect_tx(bar, STAGE_BYTES);
    bulk_load(st, S + sh * (DK * DV), STATE_BYTES, bar);
    bulk_load(st + STATE_BYTES, q + sh * DK, VEC_BYTES, bar);
    bulk_load(st + STATE_BYTES + VEC_BYTES, k + sh * DK, VEC_BYTES, bar);
    bulk_load(st + STATE_BYTES + 2 * VEC_BYTES, v + sh * DV, VEC_BYTES, bar);
    if (CG) bulk_load(st + STATE_BYTES + 3 * VEC_BYTES, a + sh * DK, GATE_VEC_BYTES, bar);
  };
  int issued = 0;
  if (tid == 0) {
    for (; issued < min(2, n_items); ++issued) issue(issued);
  }
  float a_next = 0.f, b_next = 0.f;
  if (n_items > 0) {
    a_next = CG ? 1.f : __ldg(a + first);
    b_next = __ldg(b + first);
  }
  const int r0 = warp * (DK / 8);                 // this thread: rows r0 .. r0+15, columns 4 lane .. +3
  for (int n = 0; n < n_items; ++n) {
    const long long sh = first + (long long)n * step;
    const float aa = a_next, bb = b_next;
    if (n + 1 < n_items) {                        // gates of the next item, a whole item ahead
      if (!CG) a_next = __ldg(a + sh + step);
      b_next = __ldg(b + sh + step);
    }
    uint8_t* st = dsm + (n % STAGES) * STAGE_BYTES;
    const bool okw = mbar_wait_bounded(&full[n % STAGES], (n / STAGES) & 1, abort_flag, status);
    if (__syncthreads_or(!okw || *abort_flag != 0)) break;
    float* sS = reinterpret_cast<float*>(st);
    const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(st + STATE_BYTES);
    const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(st + STATE_BYTES + VEC_BYTES);
    const __nv_bfloat16* sv = reinterpret_cast<const __nv_bfloat16*>(st + STATE_BYTES + 2 * VEC_BYTES);
    const float* sa = reinterpret_cast<const float*>(st + STATE_BYTES + 3 * VEC_BYTES);   // CG only
    // norms and k.q over the whole vectors (every warp, no block sync needed)
    float qq = 0.f, kk = 0.f, kq = 0.f;
#pragma unroll
    for (int e = 0; e < DK / 32; ++e) {
      const float qe = __bfloat162float(sq[lane + 32 * e]);
      const float ke = __bfloat162float(sk[lane + 32 * e]);
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
    // this thread's 16 x 4 block of the state, and its partial x_k, x_q
    float s[DK / 8][4], kr[DK / 8], ar[DK / 8];
    float xk[4] = {0.f, 0.f, 0.f, 0.f}, xq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < DK / 8; ++i) {
      const float4 t = *reinterpret_cast<const float4*>(sS + (r0 + i) * DV + 4 * lane);
      s[i][0] = t.x, s[i][1] = t.y, s[i][2] = t.z, s[i][3] = t.w;
      kr[i] = __bfloat162float(sk[r0 + i]) * nk;
      ar[i] = CG ? sa[r0 + i] : aa;
      const float qr = __bfloat162float(sq[r0 + i]) * nq;
      const float kw = CG ? kr[i] * ar[i] : kr[i];
      const float qw = CG ? qr * ar[i] : qr;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        xk[c] = fmaf(s[i][c], kw, xk[c]);
        xq[c] = fmaf(s[i][c], qw, xq[c]);
      }
    }
    *reinterpret_cast<float4*>(red + (warp * 2 + 0) * DV + 4 * lane) = make_float4(xk[0], xk[1], xk[2], xk[3]);
    *reinterpret_cast<float4*>(red + (warp * 2 + 1) * DV + 4 * lane) = make_float4(xq[0], xq[1], xq[2], xq[3]);
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 4; ++c) xk[c] = xq[c] = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float4 pk = *reinterpret_cast<const float4*>(red + (w * 2 + 0) * DV + 4 * lane);
      const float4 pq = *reinterpret_cast<const float4*>(red + (w * 2 + 1) * DV + 4 * lane);
      xk[0] += pk.x, xk[1] += pk.y, xk[2] += pk.z, xk[3] += pk.w;
      xq[0] += pq.x, xq[1] += pq.y, xq[2] += pq.z, xq[3] += pq.w;
    }
    const float kqn = kq * nk * nq;
    float u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) u[c] = bb * (__bfloat162float(sv[4 * lane + c]) - aa * xk[c]);
    if (warp == 0) {
      float y[4];
      const float og = gate_factor(ep, sh);
#pragma unroll
      for (int c = 0; c < 4; ++c) y[c] = og * (scale * fmaf(aa, xq[c], kqn * u[c]));
      uint2 ov;
      if (ep.h_prev) {
        const uint2 hp = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(ep.h_prev) +
                                                         sh * DV + 4 * lane);
        const float4 r = __ldg(reinterpret_cast<const float4*>(ep.rho + (sh % ep.H) * DV + 4 * lane));
        // o rounded to bf16 first, as loop_residual would see it
        ov.x = pack_bf16x2(fmaf(r.x, bf16_lo(hp.x), to_f32(from_f32<__nv_bfloat16>(y[0]))),
                           fmaf(r.y, bf16_hi(hp.x), to_f32(from_f32<__nv_bfloat16>(y[1]))));
        ov.y = pack_bf16x2(fmaf(r.z, bf16_lo(hp.y), to_f32(from_f32<__nv_bfloat16>(y[2]))),
                           fmaf(r.w, bf16_hi(hp.y), to_f32(from_f32<__nv_bfloat16>(y[3]))));
      } else {
        ov.x = pack_bf16x2(y[0], y[1]);
        ov.y = pack_bf16x2(y[2], y[3]);
      }
      *reinterpret_cast<uint2*>(o + sh * DV + 4 * lane) = ov;
    }
#pragma unroll
    for (int i = 0; i < DK / 8; ++i) {
      float4 t;
      t.x = fmaf(ar[i], s[i][0], kr[i] * u[0]);
      t.y = fmaf(ar[i], s[i][1], kr[i] * u[1]);
      t.z = fmaf(ar[i], s[i][2], kr[i] * u[2]);
      t.w = fmaf(ar[i], s[i][3], kr[i] * u[3]);
      *reinterpret_cast<float4*>(sS + (r0 + i) * DV + 4 * lane) = t;
    }
    fence_proxy_async_smem();
    __syncthreads();        // the new state is in the stage; every read of red is done
    if (tid == 0) {
      bulk_store(S + sh * (DK * DV), sS, STATE_BYTES);
      if (issued < n_items) {
        // item n+2 goes into the stage of item n-1, whose store has read it by now
        bulk_wait_read<1>();
        issue(issued);
        ++issued;
      }
    }
  }
  if (tid == 0) {
    // leave no bulk copy in flight: loads issued but not consumed, and stores
    for (int n = 0; n < issued; ++n) {
      if (n >= issued - STAGES)
        mbar_wait_bounded(&full[n % STAGES], (n / STAGES) & 1, nullptr, status);
    }
    bulk_wait_all();
  }
  __syncthreads();
}
}  // namespace dec

template <int DK, typename T, bool CG>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* a,
                                   const float* b, float* S, void* o, long long NH, int dv,
                                   float scale, unsigned flags, const Epilogue& ep, cudaStream_t stream) {
  const bool wide = (dv % 128) == 0;
  const int cols = wide ? 128 : 64;
  const long long blocks = NH * (dv / cols);
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (wide)
    gdn_decode_kernel<DK, 4, T, CG><<<(unsigned)blocks, 256, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, a, b, S, (T*)o, dv, scale, flags, ep);
  else
    gdn_decode_kernel<DK, 2, T, CG><<<(unsigned)blocks, 256, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, a, b, S, (T*)o, dv, scale, flags, ep);
  return cudaGetLastError();
}

template <bool CG>
static cudaError_t launch_stream(const void* q, const void* k, const void* v, const float* a,
                                 const float* b, float* S, void* o, long long NH, float scale,
                                 unsigned flags, int num_sms, unsigned* status, const Epilogue& ep,
                                 cudaStream_t stream) {
  static std::atomic<bool> attr_set[kMaxDevices];
  const cudaError_t e = smem_attr_once(attr_set, dec::gdn_decode_stream_kernel<CG>, dec::Ring<CG>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long blocks = NH < num_sms ? NH : num_sms;
  dec::gdn_decode_stream_kernel<CG><<<(unsigned)blocks, dec::THREADS, dec::Ring<CG>::SMEM_BYTES, stream>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, a, b, S,
      (__nv_bfloat16*)o, NH, scale, flags, status, ep);
  return cudaGetLastError();
}

template <bool CG>
static cudaError_t launch_decode_cg(const void* q, const void* k, const void* v, const float* a,
                                    const float* b, float* S, void* o, long long NH, int dk, int dv,
                                    gdn_dtype dt, float scale, unsigned flags, int num_sms,
                                    unsigned* status, const Epilogue& ep, cudaStream_t stream) {
  if (dt == GDN_BF16 && dk == dec::DK && dv == dec::DV && status)
    return launch_stream<CG>(q, k, v, a, b, S, o, NH, scale, flags, num_sms, status, ep, stream);
  if (dt == GDN_BF16) {
    return dk == 128 ? launch_decode_t<128, __nv_bfloat16, CG>(q, k, v, a, b, S, o, NH, dv, scale, flags, ep, stream)
                     : launch_decode_t<64, __nv_bfloat16, CG>(q, k, v, a, b, S, o, NH, dv, scale, flags, ep, stream);
  }
  return dk == 128 ? launch_decode_t<128, float, CG>(q, k, v, a, b, S, o, NH, dv, scale, flags, ep, stream)
                   : launch_decode_t<64, float, CG>(q, k, v, a, b, S, o, NH, dv, scale, flags, ep, stream);
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* a,
                          const float* b, float* S, void* o, const float* gate, const void* h_prev,
                          const float* rho, int N, int H, int dk, int dv, gdn_dtype dt, float scale,
                          unsigned flags, int num_sms, unsigned* status, cudaStream_t stream) {
  const long long NH = (long long)N * H;
  const Epilogue ep{gate, h_prev, rho, H};
  if (NH == 0) return cudaSuccess;
  if (flags & GDN_CHANNEL_GATE)
    return launch_decode_cg<true>(q, k, v, a, b, S, o, NH, dk, dv, dt, scale, flags, num_sms, status, ep, stream);
  return launch_decode_cg<false>(q, k, v, a, b, S, o, NH, dk, dv, dt, scale, flags, num_sms, status, ep, stream);
}

}  // namespace gdn
