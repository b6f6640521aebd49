// Per-loop learned residual of a looped linear-time transformer
// ("LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph):
//     h^(tau) = h~^(tau) + rho_tau (.) h^(tau-1),   rho_tau in R^d per channel.
//
// HBM-bound elementwise pass (6 bytes per bf16 element: two reads, one write).
// Each thread moves 16-byte vectors (8 bf16 or 4 fp32); the grid is a multiple
// of the SM count and strides over the tensor.  h_out may alias either input:
// every element is read and then written by the same thread only.
#include "common.cuh"

namespace gdn {

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__global__ void __launch_bounds__(256) loop_residual_bf16_kernel(
    const uint4* h_tilde, const uint4* h_prev,
    const float* __restrict__ rho, uint4* h_out, int64_t n_vec, int d) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
    const uint4 x = ld_stream(h_tilde + i);
    const uint4 y = ld_stream(h_prev + i);
    const int c0 = (int)((i * 8) % d);
    const float4 r0 = __ldg(reinterpret_cast<const float4*>(rho + c0));
    const float4 r1 = __ldg(reinterpret_cast<const float4*>(rho + c0 + 4));
    uint4 o;
    o.x = pack_bf16x2(fmaf(r0.x, bf16_lo(y.x), bf16_lo(x.x)), fmaf(r0.y, bf16_hi(y.x), bf16_hi(x.x)));
    o.y = pack_bf16x2(fmaf(r0.z, bf16_lo(y.y), bf16_lo(x.y)), fmaf(r0.w, bf16_hi(y.y), bf16_hi(x.y)));
    o.z = pack_bf16x2(fmaf(r1.x, bf16_lo(y.z), bf16_lo(x.z)), fmaf(r1.y, bf16_hi(y.z), bf16_hi(x.z)));
    o.w = pack_bf16x2(fmaf(r1.z, bf16_lo(y.w), bf16_lo(x.w)), fmaf(r1.w, bf16_hi(y.w), bf16_hi(x.w)));
    __stcs(h_out + i, o);
  }
}

__global__ void __launch_bounds__(256) loop_residual_f32_kernel(
    const float4* h_tilde, const float4* h_prev,
    const float* __restrict__ rho, float4* h_out, int64_t n_vec, int d) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
    const uint4 xu = ld_stream(h_tilde + i);
    const uint4 yu = ld_stream(h_prev + i);
    const int c0 = (int)((i * 4) % d);
    const float4 r = __ldg(reinterpret_cast<const float4*>(rho + c0));
    float4 o;
    o.x = fmaf(r.x, __uint_as_float(yu.x), __uint_as_float(xu.x));
    o.y = fmaf(r.y, __uint_as_float(yu.y), __uint_as_float(xu.y));
    o.z = fmaf(r.z, __uint_as_float(yu.z), __uint_as_float(xu.z));
    o.w = fmaf(r.w, __uint_as_float(yu.w), __uint_as_float(xu.w));
    __stcs(h_out + i, o);
  }
}

cudaError_t launch_loop_residual(const void* h_tilde, const void* h_prev, const float* rho,
                                 void* h_out, int64_t rows, int d, gdn_dtype dt, int num_sms,
                                 cudaStream_t stream) {
  const int64_t elems = rows * (int64_t)d;
  const int per_vec = (dt == GDN_BF16) ? 8 : 4;
  const int64_t n_vec = elems / per_vec;
  if (n_vec == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (n_vec + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 8;   // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  if (dt == GDN_BF16) {
    loop_residual_bf16_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const uint4*>(h_tilde), static_cast<const uint4*>(h_prev), rho,
        static_cast<uint4*>(h_out), n_vec, d);
  } else {
    loop_residual_f32_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const float4*>(h_tilde), static_cast<const float4*>(h_prev), rho,
        static_cast<float4*>(h_out), n_vec, d);
  }
  return cudaGetLastError();
}

}  // namespace gdn
