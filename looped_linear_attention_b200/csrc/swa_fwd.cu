// Sliding-window causal softmax attention on the 5th-generation tensor cores
// (tcgen05 MMA with tensor-memory accumulators, TMA-fed shared memory), sm_100a.
//
// The window mixer of the hybrid LT2 loops ("LT2: Linear-Time Looped
// Transformers", §2: a sliding-window block of window w, whose receptive
// field grows to T w over T loops; Appendix C: the windowed variants attend to
// the w - 1 previous tokens and the token itself, none after it).  For query
// t of a sequence starting at t0, over the keys j in [max(t0, t - w + 1), t]:
//     o_t = sum_j softmax_j(scale q_t . k_j) v_j.
//
// One CTA per (sequence, head, tile of 128 queries) walks the 128-key tiles
// that the tile's windows touch, flash-attention style, with its warps
// specialised:
//   * a control warp issues every TMA load (Q once; K and V tiles through two
//     buffers each, in the 128-byte swizzle) and every tcgen05 MMA: S = Q K^T
//     into one of two tensor-memory S buffers, O += P V into the O columns
//     (M = 128 queries, N = 128, K = 128), each committed to an mbarrier;
//   * eight softmax warps, two threads per query row r (tensor-memory lane r,
//     warps w and w + 4, one per half of the 128 keys): each loads its half
//     of the S row once, masks it to the row's window (tiles inside every
//     row's window skip the mask), and the two exchange their partial maxima
//     through a 64-thread named barrier of the pair; the running maximum m is
//     kept in base 2, each thread keeps its partial sum of P = 2^(s - m),
//     writes its half of P into one of two P buffers (the bf16 A operand) and
//     its warp arrives on that buffer's mbarrier; O is rescaled in tensor
//     memory only when the maximum grew by more than 2^8 (otherwise the stale
//     maximum keeps every P <= 2^8; the result is the same after the final
//     division by l).
// Hand-offs are mbarriers, so the softmax of tile t runs while the tensor
// cores compute P V of tile t - 1 and S of tile t + 1: S_{t+2} is issued once
// the softmax has read S_t, K_{t+2} loaded once S_t is done, V_{t+1} once
// P V of tile t - 1 is done, and P_t written once P V of tile t - 2 is done.
// Every wait is bounded (GDN_ERR_TIMEOUT).  The epilogue divides by l and
// stores bf16 rows, staged through shared memory for 16-byte coalesced stores.
#include "common.cuh"
#include "tma_host.h"

namespace gdn {
namespace swa {

constexpr int D = 128;        // head width of q, k and v
constexpr int BM = 128;       // queries per CTA
constexpr int BN = 128;       // keys per tile
constexpr int SOFTMAX_THREADS = 256;               // two threads per query row
constexpr int THREADS = SOFTMAX_THREADS + 32;      // + the control warp
constexpr int CONTROL_WARP = SOFTMAX_THREADS / 32;
constexpr uint32_t TILE_BYTES = 32768;           // 128 rows x 128 bf16, two 64-column slabs
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE_BYTES;      // 2 buffers
constexpr uint32_t OFF_V = OFF_K + 2 * TILE_BYTES;  // 2 buffers
constexpr uint32_t OFF_P = OFF_V + 2 * TILE_BYTES;  // 2 buffers of P (bf16 A operand); output staging
constexpr uint32_t OFF_RED = OFF_P + 2 * TILE_BYTES;  // [2 tiles][2 halves][128 rows] fp32 maxima / sums
constexpr uint32_t OFF_OKF = OFF_RED + 2 * 2 * BM * 4;  // [2 tiles][8 warps] int: the warp is still on track
constexpr uint32_t OFF_BAR = OFF_OKF + 2 * 8 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds 227 KB");
// tensor-memory columns: S (two buffers) and O
constexpr uint32_t COL_S = 0;
constexpr uint32_t COL_O = 256;
constexpr uint32_t TMEM_COLS = 512;

// mbarriers: Q; K, V, S, P (count 8: one arrival per softmax warp), O (P V done): two each
enum : int { B_Q = 0, B_K = 1, B_V = 3, B_S = 5, B_P = 7, B_O = 9, NBAR = 11 };
static_assert(8 * NBAR + 8 <= 128, "barrier area");

struct Params {
  __nv_bfloat16* o;
  const int32_t* cu_seqlens;
  unsigned* status;
  int n_seq, seq_len, max_seq_len, total_tokens, H, window;
  float scale_log2;   // scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return smem_desc(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr, uint32_t lbo) { return smem_desc(saddr, lbo, 1024); }
// Two 32-column loads (columns at taddr0 and taddr1 of the warp's 32 lanes)
// under one wait: v[0..31] from taddr0, v[32..63] from taddr1.
__device__ __forceinline__ void tmem_ld32x2(uint32_t taddr0, uint32_t taddr1, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr0), "r"(taddr1)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}
// Named barriers: 1 + quad for the two warps of a query-row block (64
// threads), 5 for the eight softmax warps.
__device__ __forceinline__ void pair_sync(int quad) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + quad) : "memory");
}
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 5, 256;" ::: "memory"); }

// One 128 x 128 tile (tokens tok0 .. tok0 + 127 of head h) in two 64-column slabs.
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int h,
                                          int tok0) {
  mbar_arrive_expect_tx(bar, TILE_BYTES);
  tma_load_3d(dst, map, bar, 0, h, tok0);
  tma_load_3d(dst + 8192, map, bar, 0, h, tok0 + 64);
  tma_load_3d(dst + 16384, map, bar, 64, h, tok0);
  tma_load_3d(dst + 24576, map, bar, 64, h, tok0 + 64);
}

__global__ void __launch_bounds__(THREADS, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(sm) & 1023u) {
    if (tid == 0) record_status(p.status, GDN_ERR_CUDA);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8 * NBAR);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_BAR + 8 * NBAR + 4);
  volatile int* s_okf = reinterpret_cast<volatile int*>(sm + OFF_OKF);

  // block -> (sequence, head, query tile); query tiles fastest so that
  // neighbouring CTAs share K and V tiles in L2, last tiles first (they have
  // the most key tiles: the longest blocks start in the first wave)
  const int n_qt = (p.max_seq_len + BM - 1) / BM;
  const int qt = n_qt - 1 - (int)(blockIdx.x % n_qt);
  const int h = (blockIdx.x / n_qt) % p.H;
  const int seq = blockIdx.x / (n_qt * p.H);
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
    bool bad = (s0 != seq_start || s1 != seq_end);
    // a sequence longer than max_seq_len would lose its last queries
    bad = bad || (qt == n_qt - 1 && s1 - s0 > p.max_seq_len);
    if (bad && tid == 0) record_status(p.status, GDN_ERR_INVALID);
    seq_start = s0;
    seq_end = s1;
  }
  const int q0 = seq_start + qt * BM;
  if (q0 >= seq_end) return;                       // past this sequence (uniform per CTA)
  // key tiles (128 keys from the sequence start) touched by the windows of this tile
  const int key_lo = max(seq_start, q0 - p.window + 1);
  const int key_hi = min(q0 + BM - 1, seq_end - 1);
  const int t_first = (key_lo - seq_start) / BN;
  const int n_tiles = (key_hi - seq_start) / BN - t_first + 1;
  auto key_tok = [&](int t) { return seq_start + (t_first + t) * BN; };

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], (i == B_P || i == B_P + 1) ? 8 : 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == CONTROL_WARP) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = smem_u32(sm);

  if (warp == CONTROL_WARP) {
    // ================= control warp: loads and MMAs
    int k_issued = 0, v_issued = 0;                // tiles whose K / V loads lane 0 issued
    int s_issued = 0, pv_issued = 0;               // S and P V products issued
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      load_tile(sm + OFF_Q, &tm_q, &bars[B_Q], h, q0);
    }
    for (; k_issued < min(2, n_tiles); ++k_issued)
      if (lane == 0)
        load_tile(sm + OFF_K + k_issued * TILE_BYTES, &tm_k, &bars[B_K + k_issued], h, key_tok(k_issued));
    for (; v_issued < min(2, n_tiles); ++v_issued)
      if (lane == 0)
        load_tile(sm + OFF_V + v_issued * TILE_BYTES, &tm_v, &bars[B_V + v_issued], h, key_tok(v_issued));
    __syncwarp();
    auto wait = [&](int bar, int parity) -> bool {
      const bool okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[bar], parity, s_abort, p.status));
      tc_fence_after();
      return okw;
    };
    // S_t = Q K_t^T into S buffer t % 2
    auto issue_s = [&](int t) {
      if (elect_one()) {
        const uint32_t kt = sbase + OFF_K + (t & 1) * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(tmem + COL_S + (t & 1) * BN, kdesc(sbase + OFF_Q + off), kdesc(kt + off),
                   idesc_bf16(128, 128, 0, 0), kk > 0);
        }
        mma_commit(&bars[B_S + (t & 1)]);
      }
      __syncwarp();
      ++s_issued;
    };
    bool okc = wait(B_Q, 0) && wait(B_K, 0);
    if (okc) issue_s(0);
    if (okc && n_tiles > 1 && (okc = wait(B_K + 1, 0))) issue_s(1);
    for (int t = 0; t < n_tiles && okc; ++t) {
      // K_{t+2} into the buffer S_t has finished reading
      if (t + 2 < n_tiles) {
        if (!(okc = wait(B_S + (t & 1), (t >> 1) & 1))) break;
        if (lane == 0) load_tile(sm + OFF_K + (t & 1) * TILE_BYTES, &tm_k, &bars[B_K + (t & 1)], h, key_tok(t + 2));
        ++k_issued;
      }
      // V_{t+1} into the buffer P V of tile t - 1 has finished reading
      if (t >= 1 && t + 1 < n_tiles && v_issued == t + 1) {
        if (!(okc = wait(B_O + ((t - 1) & 1), ((t - 1) >> 1) & 1))) break;
        if (lane == 0)
          load_tile(sm + OFF_V + ((t + 1) & 1) * TILE_BYTES, &tm_v, &bars[B_V + ((t + 1) & 1)], h, key_tok(t + 1));
        ++v_issued;
      }
      // O += P_t V_t once the softmax warps have written P_t
      if (!(okc = wait(B_P + (t & 1), (t >> 1) & 1) && wait(B_V + (t & 1), (t >> 1) & 1))) break;
      if (elect_one()) {
        const uint32_t vt = sbase + OFF_V + (t & 1) * TILE_BYTES;
        const uint32_t pt = sbase + OFF_P + (t & 1) * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_bf16(tmem + COL_O, kdesc(pt + (kk >> 2) * 16384 + (kk & 3) * 32), mndesc(vt + kk * 2048, 16384),
                   idesc_bf16(128, 128, 0, 1), (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[B_O + (t & 1)]);
      }
      __syncwarp();
      ++pv_issued;
      // S_{t+2} into the S buffer the softmax has read (P_t written implies it)
      if (t + 2 < n_tiles) {
        if (!(okc = wait(B_K + (t & 1), ((t + 2) >> 1) & 1))) break;
        issue_s(t + 2);
      }
    }
    if (lane == 0) {
      // never leave with a bulk copy still landing in shared memory, or an MMA
      // still writing tensor memory: every load and product issued is waited
      // for (bounded; on the normal path they are long complete)
      mbar_wait_bounded(&bars[B_Q], 0, nullptr, p.status);
      for (int t = max(0, k_issued - 2); t < k_issued; ++t)
        mbar_wait_bounded(&bars[B_K + (t & 1)], (t >> 1) & 1, nullptr, p.status);
      for (int t = max(0, v_issued - 2); t < v_issued; ++t)
        mbar_wait_bounded(&bars[B_V + (t & 1)], (t >> 1) & 1, nullptr, p.status);
      for (int t = max(0, s_issued - 2); t < s_issued; ++t)
        mbar_wait_bounded(&bars[B_S + (t & 1)], (t >> 1) & 1, nullptr, p.status);
      for (int t = max(0, pv_issued - 2); t < pv_issued; ++t)
        mbar_wait_bounded(&bars[B_O + (t & 1)], (t >> 1) & 1, nullptr, p.status);
    }
    __syncwarp();
  } else {
    // ================= softmax warps
    const int quad = warp & 3, hf = warp >> 2;    // tensor-memory lane block, key / column half
    const int r = quad * 32 + lane;                // query row of this thread
    const int q_tok = q0 + r;
    const bool row_valid = q_tok < seq_end;
    const int win_lo = q_tok - p.window + 1;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float* s_red = reinterpret_cast<float*>(sm + OFF_RED);   // [tile & 1][hf][row]
    float m_run = -1e30f, l_run = 0.f;             // running maximum (base 2); this half's sum
    // tiles that lie inside every row's window (and rows all inside the
    // sequence) need no mask
    const bool rows_full = q0 + BM <= seq_end;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int kt0 = key_tok(t);
      const bool interior = rows_full && kt0 + BN - 1 <= q0 && kt0 >= q0 + BM - 1 - p.window + 1;
      // ---- S_t is in tensor memory: this thread's half of the S row (64
      // keys), scaled to base 2 and masked
      bool okw = ok && __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_S + (t & 1)], (t >> 1) & 1, s_abort,
                                                                  p.status));
      tc_fence_after();
      float x[64];
      float tmax = -INFINITY;
      if (okw) {
        const uint32_t s_col = tmem + lane_off + COL_S + (t & 1) * BN + hf * 64;
        tmem_ld32x2(s_col, s_col + 32, x);
        float pm[8];                               // eight partial maxima (short dependency chains)
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
        if (interior) {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            x[e] *= p.scale_log2;
            pm[e & 7] = fmaxf(pm[e & 7], x[e]);
          }
        } else {
          const int j0 = kt0 + hf * 64;
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            const int j = j0 + e;
            const bool in = row_valid && j <= q_tok && j >= win_lo;
            x[e] = in ? x[e] * p.scale_log2 : -INFINITY;
            pm[e & 7] = fmaxf(pm[e & 7], x[e]);
          }
        }
        tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      // ---- the row maximum from both halves (and whether both warps are on track)
      float* red = s_red + (t & 1) * 2 * BM;
      red[hf * BM + r] = tmax;
      if (lane == 0) s_okf[(t & 1) * 8 + warp] = okw ? 1 : 0;
      pair_sync(quad);
      ok = okw && s_okf[(t & 1) * 8 + (warp ^ 4)] != 0;
      if (!ok) break;                              // both warps of the pair leave together
      tmax = fmaxf(tmax, red[(hf ^ 1) * BM + r]);
      const float m_new = fmaxf(m_run, tmax);
      // lazy rescale: only when the maximum grew by more than 8 (in base 2)
      const bool grow = (t > 0) && (m_new > m_run + 8.f);
      const float alpha = grow ? ex2(m_run - m_new) : 1.f;
      if (t == 0 || grow) m_run = m_new;
      if (__any_sync(0xffffffffu, grow)) {
        // every P V so far is done before O is rescaled (the next one needs this P)
        okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_O + ((t - 1) & 1)], ((t - 1) >> 1) & 1,
                                                        s_abort, p.status));
        tc_fence_after();
        if (okw) {
          l_run *= alpha;
#pragma unroll 1
          for (int piece = 0; piece < 2; ++piece) {
            float y[32];
            const uint32_t oc = tmem + lane_off + COL_O + hf * 64 + piece * 32;
            tmem_ld32(oc, y);
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] *= alpha;
            tmem_st32(oc, y);
          }
          tmem_wait_st();
        }
      }
      // ---- P buffer t % 2 is free once P V of tile t - 2 is done
      if (okw && t >= 2)
        okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_O + (t & 1)], ((t - 2) >> 1) & 1, s_abort,
                                                        p.status));
      if (okw) {
        // ---- P = 2^(s - m) (bf16, swizzled A operand, slab hf), l += sum P
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // eight partial sums
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          x[e] = ex2(x[e] - m_run);                // masked entries: 2^-inf = 0
          ps[e & 7] += x[e];
        }
        l_run += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        uint8_t* slab = sm + OFF_P + (t & 1) * TILE_BYTES + hf * 16384;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 o;
          o.x = pack_bf16x2(x[c * 8 + 0], x[c * 8 + 1]);
          o.y = pack_bf16x2(x[c * 8 + 2], x[c * 8 + 3]);
          o.z = pack_bf16x2(x[c * 8 + 4], x[c * 8 + 5]);
          o.w = pack_bf16x2(x[c * 8 + 6], x[c * 8 + 7]);
          *reinterpret_cast<uint4*>(slab + sw128_offset(r, c * 8)) = o;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_P + (t & 1)]);
      }
      ok = okw;                                    // a failure here reaches the partner next tile
    }
    // ---- epilogue: O / l, staged through shared memory for coalesced stores
    bool okw = ok;
    if (okw && n_tiles > 0)
      okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_O + ((n_tiles - 1) & 1)],
                                                      ((n_tiles - 1) >> 1) & 1, s_abort, p.status));
    tc_fence_after();
    float* red = s_red;                            // tile slot 0 (the loop's last use of it is behind a pair barrier)
    softmax_sync();                                // no pair still reads the exchange area
    red[hf * BM + r] = l_run;                      // the two halves' sums
    if (lane == 0) s_okf[warp] = okw ? 1 : 0;
    softmax_sync();
    bool all_ok = true;
#pragma unroll
    for (int w = 0; w < 8; ++w) all_ok = all_ok && s_okf[w] != 0;
    uint8_t* stage = sm + OFF_P;                   // [128 rows][256 B], 16-byte chunks XOR-swizzled
    if (all_ok) {
      const float l = l_run + red[(hf ^ 1) * BM + r];
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int piece = 0; piece < 2; ++piece) {
        float y[32];
        tmem_ld32(tmem + lane_off + COL_O + hf * 64 + piece * 32, y);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 o;
          o.x = pack_bf16x2(y[c * 8 + 0] * inv, y[c * 8 + 1] * inv);
          o.y = pack_bf16x2(y[c * 8 + 2] * inv, y[c * 8 + 3] * inv);
          o.z = pack_bf16x2(y[c * 8 + 4] * inv, y[c * 8 + 5] * inv);
          o.w = pack_bf16x2(y[c * 8 + 6] * inv, y[c * 8 + 7] * inv);
          const int chunk = hf * 8 + piece * 4 + c;
          *reinterpret_cast<uint4*>(stage + r * 256 + ((chunk ^ (r & 15)) * 16)) = o;
        }
      }
    }
    softmax_sync();
    if (all_ok) {
      const int rows = min(BM, seq_end - q0);
#pragma unroll 4
      for (int it = tid; it < BM * 16; it += SOFTMAX_THREADS) {
        const int i = it >> 4, chunk = it & 15;
        if (i < rows) {
          const uint4 v = *reinterpret_cast<const uint4*>(stage + i * 256 + ((chunk ^ (i & 15)) * 16));
          __stcs(reinterpret_cast<uint4*>(p.o + ((size_t)(q0 + i) * p.H + h) * D + chunk * 8), v);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == CONTROL_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace swa

gdn_status launch_swa(const swa_params* p, unsigned* status, cudaStream_t stream) {
  static std::atomic<bool> attr_set[kMaxDevices];
  if (smem_attr_once(attr_set, swa::swa_fwd_kernel, swa::SMEM_BYTES) != cudaSuccess) return GDN_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, p->q, swa::D, p->H, p->total_tokens) || !make_map(&mk, p->k, swa::D, p->H, p->total_tokens) ||
      !make_map(&mv, p->v, swa::D, p->H, p->total_tokens))
    return GDN_ERR_CUDA;
  swa::Params kp;
  kp.o = static_cast<__nv_bfloat16*>(p->o);
  kp.cu_seqlens = p->cu_seqlens;
  kp.status = status;
  kp.n_seq = p->n_seq;
  kp.seq_len = p->seq_len;
  kp.max_seq_len = p->cu_seqlens ? p->max_seq_len : p->seq_len;
  kp.total_tokens = p->total_tokens;
  kp.H = p->H;
  kp.window = p->window;
  kp.scale_log2 = p->scale * 1.4426950408889634f;
  const long long blocks = (long long)p->n_seq * p->H * ((kp.max_seq_len + swa::BM - 1) / swa::BM);
  if (blocks <= 0) return GDN_OK;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  swa::swa_fwd_kernel<<<(unsigned)blocks, swa::THREADS, swa::SMEM_BYTES, stream>>>(mq, mk, mv, kp);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace gdn
