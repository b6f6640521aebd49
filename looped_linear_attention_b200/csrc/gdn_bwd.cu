// Reverse mode of the gated delta rule (gdn_chunk_bwd): gradients with respect
// to q, k, v, a, b and S0 of a loss that depends on the outputs and the final
// states.  The recurrence ("LT2: Linear-Time Looped Transformers", §2, in the
// dk x dv orientation) is
//     S_t = a_t (S_{t-1} - b_t k_t x_t^T) + b_t k_t v_t^T,   x_t = S_{t-1}^T k_t,
//     o_t = scale S_t^T q_t,
// and its reverse mode, token by token backwards with G_t = dloss/dS_t:
//     G_t      = dS_t + scale q_t do_t^T,          y_t = G_t^T k_t
//     dq_t     = scale S_t do_t                    dv_t = b_t y_t
//     dk_t     = -a_t b_t (G_t x_t + S_{t-1} y_t) + b_t G_t v_t
//     da_t     = <G_t, S_{t-1}> - b_t y_t . x_t    db_t = y_t . (v_t - a_t x_t)
//     dS_{t-1} = a_t (G_t - b_t k_t y_t^T).
//
// First implementation, fp32 on the CUDA cores: one CTA per (sequence, head)
// chain.  A forward pass writes the state every 64 tokens (a checkpoint);
// then, chunk by chunk from the end, the chunk's 65 states are recomputed from
// its checkpoint and its tokens are walked backwards.  States, checkpoints and
// G live in the workspace ([dk][dv] fp32 each, L1/L2-resident while in use).
// Column-parallel work (the state steps, G, x, y, dv, the da/db partial sums)
// gives thread j column j; row-parallel work (dq, dk) gives thread i row i.
#include "common.cuh"

namespace gdn {
namespace bwd {

constexpr int C = 64;            // checkpoint interval (tokens)
constexpr int THREADS = 256;     // >= dv (columns) and >= dk (rows)
constexpr int MAX_DIM = 256;

struct KParams {
  const void *q, *k, *v, *go;
  const float *a, *b, *S0, *gST;
  float *gq, *gk, *gv, *ga, *gb, *gS0;
  const int32_t* cu;
  int n_seq, seq_len, total, H, dk, dv;
  float scale;
  float *ckpt, *states, *G;
  long long ckpt_slots;            // checkpoint slots per head
  unsigned* status;
};

__device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

template <typename T>
__global__ void __launch_bounds__(THREADS, 1) gdn_bwd_kernel(const KParams p) {
  __shared__ float sk[MAX_DIM], sq[MAX_DIM], sv[MAX_DIM], sgo[MAX_DIM];
  __shared__ float sx[MAX_DIM], sy[MAX_DIM], spa[MAX_DIM], spb[MAX_DIM];
  const int tid = threadIdx.x;
  const int chain = blockIdx.x;
  const int s = chain / p.H, h = chain % p.H;
  const int dk = p.dk, dv = p.dv;
  const size_t sd = (size_t)dk * dv;
  int t0, t1;
  if (p.cu) {
    t0 = p.cu[s];
    t1 = p.cu[s + 1];
  } else {
    t0 = s * p.seq_len;
    t1 = t0 + p.seq_len;
  }
  {
    // offsets outside [0, total] or decreasing: clamp, and report
    const int c0 = min(max(t0, 0), p.total);
    const int c1 = min(max(t1, c0), p.total);
    if ((c0 != t0 || c1 != t1) && tid == 0) record_status(p.status, GDN_ERR_INVALID);
    t0 = c0;
    t1 = c1;
  }
  const int n_chunks = (t1 - t0 + C - 1) / C;
  // this chain's checkpoints: slots t0 / C + 2 s .. + n_chunks - 1 of its head
  // (sequence s needs at most ceil(len / C) slots, and consecutive sequences'
  // bases differ by at least that plus one)
  float* ck = p.ckpt + ((size_t)h * p.ckpt_slots + (size_t)(t0 / C + 2 * s)) * sd;
  float* S = p.states + (size_t)chain * (C + 1) * sd;   // S[u], u = 0 .. C
  float* G = p.G + (size_t)chain * sd;
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* go = static_cast<const T*>(p.go);
  const size_t sbase = ((size_t)s * p.H + h) * sd;

  auto load_token = [&](int t) {
    const size_t th = (size_t)t * p.H + h;
    if (tid < dk) {
      sk[tid] = ld(k, th * dk + tid);
      sq[tid] = ld(q, th * dk + tid);
    }
    if (tid < dv) {
      sv[tid] = ld(v, th * dv + tid);
      sgo[tid] = ld(go, th * dv + tid);
    }
  };
  // column tid of dst = one step of the recurrence applied to src (in place allowed)
  auto step_column = [&](const float* src, float* dst, float a, float b) {
    float x = 0.f;
    for (int i = 0; i < dk; ++i) x = fmaf(sk[i], src[(size_t)i * dv + tid], x);
    const float bv = b * sv[tid];
    for (int i = 0; i < dk; ++i) {
      const float w = src[(size_t)i * dv + tid];
      dst[(size_t)i * dv + tid] = fmaf(a, w - b * sk[i] * x, sk[i] * bv);
    }
  };

  // ---- forward pass: checkpoint c = state before chunk c (working state S[0])
  if (tid < dv)
    for (int i = 0; i < dk; ++i) S[(size_t)i * dv + tid] = p.S0 ? p.S0[sbase + (size_t)i * dv + tid] : 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    __syncthreads();
    if (tid < dv)
      for (int i = 0; i < dk; ++i) ck[(size_t)c * sd + (size_t)i * dv + tid] = S[(size_t)i * dv + tid];
    const int tb = t0 + c * C, te = min(t1, tb + C);
    for (int t = tb; t < te; ++t) {
      __syncthreads();                               // the previous token's values are consumed
      load_token(t);
      __syncthreads();
      const size_t th = (size_t)t * p.H + h;
      if (tid < dv) step_column(S, S, p.a[th], p.b[th]);
    }
  }

  // ---- backward pass
  __syncthreads();
  if (tid < dv)
    for (int i = 0; i < dk; ++i) G[(size_t)i * dv + tid] = p.gST ? p.gST[sbase + (size_t)i * dv + tid] : 0.f;
  for (int c = n_chunks - 1; c >= 0; --c) {
    const int tb = t0 + c * C, n = min(t1, tb + C) - tb;
    __syncthreads();
    if (tid < dv)
      for (int i = 0; i < dk; ++i) S[(size_t)i * dv + tid] = ck[(size_t)c * sd + (size_t)i * dv + tid];
    for (int u = 0; u < n; ++u) {                    // S[u + 1] = step(S[u])
      __syncthreads();
      load_token(tb + u);
      __syncthreads();
      const size_t th = (size_t)(tb + u) * p.H + h;
      if (tid < dv) step_column(S + (size_t)u * sd, S + (size_t)(u + 1) * sd, p.a[th], p.b[th]);
    }
    for (int u = n - 1; u >= 0; --u) {
      const int t = tb + u;
      const size_t th = (size_t)t * p.H + h;
      const float at = p.a[th], bt = p.b[th];
      __syncthreads();
      load_token(t);
      __syncthreads();
      const float* St = S + (size_t)(u + 1) * sd;    // S_t
      const float* Sp = S + (size_t)u * sd;          // S_{t-1}
      // columns: G_t = dS_t + scale q do^T; x, y; dv; partial sums of da, db
      if (tid < dv) {
        const int j = tid;
        const float sgoj = p.scale * sgo[j];
        float x = 0.f, y = 0.f, gs = 0.f;
        for (int i = 0; i < dk; ++i) {
          const float g = fmaf(sq[i], sgoj, G[(size_t)i * dv + j]);
          G[(size_t)i * dv + j] = g;
          const float sp = Sp[(size_t)i * dv + j];
          y = fmaf(sk[i], g, y);
          x = fmaf(sk[i], sp, x);
          gs = fmaf(g, sp, gs);
        }
        sx[j] = x;
        sy[j] = y;
        p.gv[th * dv + j] = bt * y;
        spa[j] = gs - bt * y * x;
        spb[j] = y * (sv[j] - at * x);
      }
      __syncthreads();
      // rows: dq, dk
      if (tid < dk) {
        const int i = tid;
        float dq = 0.f, gx = 0.f, sy_ = 0.f, gv = 0.f;
        for (int j = 0; j < dv; ++j) {
          const float g = G[(size_t)i * dv + j];
          dq = fmaf(St[(size_t)i * dv + j], sgo[j], dq);
          gx = fmaf(g, sx[j], gx);
          sy_ = fmaf(Sp[(size_t)i * dv + j], sy[j], sy_);
          gv = fmaf(g, sv[j], gv);
        }
        p.gq[th * dk + i] = p.scale * dq;
        p.gk[th * dk + i] = -at * bt * (gx + sy_) + bt * gv;
      }
      if (tid >= THREADS - 32) {                     // da, db: sums of the column partials
        const int l = tid - (THREADS - 32);
        float sa = 0.f, sb = 0.f;
        for (int j = l; j < dv; j += 32) {
          sa += spa[j];
          sb += spb[j];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sa += __shfl_xor_sync(0xffffffffu, sa, off);
          sb += __shfl_xor_sync(0xffffffffu, sb, off);
        }
        if (l == 0) {
          p.ga[th] = sa;
          p.gb[th] = sb;
        }
      }
      __syncthreads();
      // columns: dS_{t-1} = a (G_t - b k y^T)
      if (tid < dv) {
        const int j = tid;
        const float byj = bt * sy[j];
        for (int i = 0; i < dk; ++i) G[(size_t)i * dv + j] = at * (G[(size_t)i * dv + j] - sk[i] * byj);
      }
    }
  }
  __syncthreads();
  if (p.gS0 && tid < dv)
    for (int i = 0; i < dk; ++i) p.gS0[sbase + (size_t)i * dv + tid] = G[(size_t)i * dv + tid];
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static long long ckpt_slots(const gdn_bwd_params* p) {
  return (long long)p->total_tokens / C + 2LL * p->n_seq + 1;
}

}  // namespace bwd

size_t bwd_workspace(const gdn_bwd_params* p) {
  const size_t sd = (size_t)p->dk * p->dv * sizeof(float);
  const size_t chains = (size_t)p->n_seq * p->H;
  return bwd::align256((size_t)p->H * bwd::ckpt_slots(p) * sd) + bwd::align256(chains * (bwd::C + 1) * sd) +
         bwd::align256(chains * sd);
}

gdn_status launch_bwd(const gdn_bwd_params* p, unsigned* status, void* ws, cudaStream_t stream) {
  const long long chains = (long long)p->n_seq * p->H;
  if (chains <= 0) return GDN_OK;
  if (chains > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  const size_t sd = (size_t)p->dk * p->dv * sizeof(float);
  bwd::KParams kp;
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
  kp.dk = p->dk;
  kp.dv = p->dv;
  kp.scale = p->scale;
  kp.ckpt_slots = bwd::ckpt_slots(p);
  char* w = static_cast<char*>(ws);
  kp.ckpt = reinterpret_cast<float*>(w);
  w += bwd::align256((size_t)p->H * kp.ckpt_slots * sd);
  kp.states = reinterpret_cast<float*>(w);
  w += bwd::align256((size_t)chains * (bwd::C + 1) * sd);
  kp.G = reinterpret_cast<float*>(w);
  kp.status = status;
  if (p->io_dtype == GDN_BF16)
    bwd::gdn_bwd_kernel<__nv_bfloat16><<<(unsigned)chains, bwd::THREADS, 0, stream>>>(kp);
  else
    bwd::gdn_bwd_kernel<float><<<(unsigned)chains, bwd::THREADS, 0, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
