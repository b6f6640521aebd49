// Chunkwise prefill of the gated delta rule on the 5th-generation tensor cores
// (tcgen05 MMA with tensor-memory accumulators, TMA-fed shared memory), sm_100a.
//
// The recurrence ("LT2: Linear-Time Looped Transformers", §2, "LT2." paragraph;
// Gated DeltaNet mixer, Appendix C), with the state Sigma in R^{dk x dv}:
//     Sigma_t = a_t (I - b_t k_t k_t^T) Sigma_{t-1} + b_t k_t v_t^T,  o_t = scale Sigma_t^T q_t.
// The page reports that LT2's GDN layers run as a fused chunkwise kernel
// (§3.2).  This file is this library's own chunked form: for a chunk of C = 64
// tokens with start state Sigma_0, g_i = sum_{j<=i} log a_j, gamma_i = exp(g_i),
// D_ij = exp(g_i - g_j) (j <= i, all <= 1):
//     A   = strict_lower(diag(b) (D o K K^T)),     T = (I + A)^{-1}
//     W   = T diag(b gamma) K,   U~ = T diag(b) V,   U = U~ - W Sigma_0
//     O   = scale (diag(gamma) Q Sigma_0 + tril(D o Q K^T) U)
//     Sigma_C = gamma_C Sigma_0 + K^T diag(gamma_C / gamma) U
// U holds the per-token corrections u_t = b_t (v_t - a_t Sigma_{t-1}^T k_t), so
// Sigma_t = a_t Sigma_{t-1} + k_t u_t^T, and the three lines above follow by
// unrolling that inside the chunk.
//
// Data path (one CTA per (sequence, head, 128-wide slice of dv); two teams of
// eight warps: a prep team builds the state-independent operands of chunk c+1
// -- A, P, T, T1, T2, U~, W^T -- while a state team runs chunk c -- the
// Sigma-dependent MMAs, the U^T operands, the state refresh and the outputs --
// and, two chunks ahead, the gate vectors, the K/Q loads and the G product.
// Each team issues its own MMAs; the hand-offs are mbarriers indexed by buffer
// slot, so no waiter can fall two phases behind):
//   * every product is issued TRANSPOSED so its M dimension is 128 (dv rows of
//     Sigma^T, dk rows of W^T, or the stacked [K; Q] rows) and lands in tensor
//     memory with lane = row: G = [K;Q] K^T, U^T = V^T T2^T - Sigma^T W^T,
//     W^T = K^T T1^T, O_A^T = Sigma^T Q^T, O_B^T = U^T P^T,
//     Sigma^T += (U^T diag(gamma_C/gamma)) K.
//   * q, k, v tiles arrive by TMA (128-byte swizzle; K and Q in a 2-stage
//     ring, V in one stage); K and V are read straight from their tiles as
//     MN-major operands.  With the q/k L2 norm the tiles stay as loaded: the
//     inverse row norms are folded into the fp32 factors that meet q and k
//     (the row and column factors of A and P, T1's column scale, the carry's
//     gamma_C / gamma and the output's gamma).  Operands computed in the CTA
//     (T1, T2, P, W^T, U^T, Sigma^T) are rounded to bf16 and written as whole
//     16-byte chunks in the same swizzled layout (W^T is an MN-major B
//     operand, so every thread writes one contiguous row).
//   * the fp32 master state stays in tensor memory for the whole sequence,
//     kept pre-multiplied by the next chunk's gamma_C so that the carry MMA
//     accumulates straight onto it; its bf16 copy in shared memory feeds the
//     next chunk's MMAs.
//   * T = (I + A)^{-1} is inverted in 16 x 16 blocks on the CUDA cores; gate
//     vectors (gamma, b gamma, gamma_C / gamma) are computed once per token.
//   * every wait is bounded (GDN_ERR_TIMEOUT) so a fault in the schedule cannot
//     hang the GPU.
#include "common.cuh"
#include "tma_host.h"

namespace gdn {
namespace tc {

constexpr int C = 64;            // chunk length
constexpr int DK = 128;          // key/query width (this kernel)
constexpr int DVS = 128;         // dv slice per CTA
constexpr int WG = 128;          // one warpgroup (tensor-memory lanes 0-127)
// warps 0-7:  prep team (state-independent part of chunk c+1); its warp 0
//             also issues the TMA loads of V (one stage)
// warps 8-15: state team (state-dependent part of chunk c); it also issues
//             the TMA loads of K and Q (two stages), folds their norms and
//             issues their G product
// Warps w and w+4 of a team reach the same 32 tensor-memory lanes (w mod 4) and
// split the columns of each row between them; 4 warps per SM sub-partition
// with up to 128 registers per thread.
constexpr int TEAM = 2 * WG;
constexpr int THREADS = 2 * TEAM;
constexpr int BAR_PREP = 1;      // named barriers of the two teams
constexpr int BAR_STATE = 2;

// tensor-memory columns (fp32 accumulators, lane = row)
constexpr uint32_t COL_GW = 0;    // [K;Q] K^T, then W^T, of a prep chunk      2 x 128 x 64 (0, 320)
constexpr uint32_t COL_U = 64;    // U^T, two buffers (chunk parity)           2 x 128 x 64
constexpr uint32_t COL_OA = 192;  // Sigma^T Q^T                                128 x 64
constexpr uint32_t COL_OB = 256;  // U^T P^T                                    128 x 64
constexpr uint32_t COL_GW1 = 320; // second G / W^T buffer                      128 x 64
constexpr uint32_t COL_S = 384;   // Sigma^T fp32 (kept pre-decayed by gamma_C) 128 x 128
constexpr uint32_t TMEM_COLS = 512;
static_assert(COL_GW + 64 <= COL_U && COL_U + 128 <= COL_OA && COL_OA + 64 <= COL_OB &&
                  COL_OB + 64 <= COL_GW1 && COL_GW1 + 64 <= COL_S && COL_S + 128 <= TMEM_COLS,
              "tensor-memory regions overlap");
__device__ __forceinline__ uint32_t col_gw(int c) { return (c & 1) ? COL_GW1 : COL_GW; }

// Shared-memory plan (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_KQ = 0;            // 2 stages x 32 KB: [K0|Q0|K1|Q1] 8 KB slabs
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t OFF_V = 65536;         // 1 stage x 16 KB: [V0|V1]
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t OFF_SIG = 81920;       // Sigma^T bf16 [128 dv][128 dk], 2 x 16 KB slabs
constexpr uint32_t OFF_WT = 114688;       // W^T bf16 [128 dk][64 tok] (MN-major B operand)
constexpr uint32_t OFF_UT = 131072;       // U^T bf16 [128 dv][64 tok]
constexpr uint32_t OFF_UTP = 147456;      // U^T diag(gamma_C/gamma) bf16; output staging
constexpr uint32_t OFF_P = 163840;        // P bf16 [64][64], two buffers (chunk parity)
constexpr uint32_t OFF_T1 = 180224;       // T diag(b gamma) bf16 [64][64]
constexpr uint32_t OFF_T2 = 188416;       // T diag(b) bf16 [64][64]
// A and T (fp32) in compact lower-block-triangular form: the ten 16 x 16 blocks
// (a, b), a >= b, each stored row-major with row stride 20 (the tf32 mma
// fragment loads of a warp then hit 32 distinct banks); blocks 324 floats apart
// so that the four diagonal blocks start in different banks.
constexpr int BLK_LD = 20;
constexpr int BLK_FLOATS = 16 * BLK_LD + 4;
__device__ __forceinline__ int blk(int a, int b) { return (a * (a + 1) / 2 + b) * BLK_FLOATS; }
constexpr uint32_t LT_BYTES = 10 * BLK_FLOATS * 4;
constexpr uint32_t OFF_A = 196608;                    // A, compact blocks
constexpr uint32_t OFF_TS = OFF_A + LT_BYTES;         // T, compact blocks (also the solve's scratch)
constexpr uint32_t OFF_GATE = OFF_TS + LT_BYTES;      // 3 buffers of gate vectors (struct Gates)
constexpr uint32_t GATE_BYTES = 11 * 64 * 4;
constexpr uint32_t OFF_BAR = OFF_GATE + 3 * GATE_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;          // tmem base, abort flag, scan carry
constexpr uint32_t SMEM_USED = OFF_MISC + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;      // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds 227 KB");
static_assert(OFF_GATE % 16 == 0 && (BLK_FLOATS * 4) % 16 == 0, "vector access alignment");

// mbarriers (index into the barrier array)
enum : int {
  B_KQ_FULL = 0,      // [2] TMA K, Q landed
  B_V_FULL = 2,       //     TMA V landed
  B_GATES = 3,        // [3] state: gate vectors of a chunk written
  B_W_READY = 6,      //     prep: U~^T and W^T of a chunk in tensor memory
  B_W_CONSUMED = 7,   //     state: W^T read out of tensor memory (its buffer is free)
  B_CHUNK_DONE = 8,   // [2] state: chunk finished (U and P buffers free)
  B_PREP_MMA = 10,    //     prep: U~ and W^T products done
  B_STATE_MMA = 11,   //     commits of the state warpgroup
  B_G_MMA = 12,       // [2] prep: G of a chunk done (by tensor-memory buffer)
  B_OA_MMA = 14,      //     state: O_A of a chunk done
  B_NEVER = 15,       //     arrived by nobody (GDN_TEST_WAIT_TIMEOUT)
  NBAR = 16
};

struct Params {
  const float* a;
  const float* b;
  const float* S0;
  float* S_T;
  __nv_bfloat16* o;
  const int32_t* cu_seqlens;
  unsigned* status;
  // epilogue of the looped block (null = off): head-wise output gate logits
  // [tokens][H] and the loop residual o += rho (.) h_prev ([tokens][H*dv], [H*dv])
  const float* gate;
  const __nv_bfloat16* h_prev;
  const float* rho;
  int n_seq, seq_len, total_tokens, H, dv, n_slices;
  float scale;
  unsigned flags;
  // Segment schedule (fixed-length sequences cut into n_segs >= 2 segments:
  // segment 0 of seg0_tok tokens, the others of seg_tok, the last one possibly
  // shorter; mode 0 runs whole sequences in one pass):
  //   mode 1: segment 0 runs in full from S0 (outputs, and its end state S_1
  //           to Sst slot 0); the CTAs after those run segments 1 .. n_segs-2
  //           from a zero state without outputs.  Their slices 0 .. n_slices-1
  //           write the segment's state contribution B_p to Bws slot p-1; one
  //           extra slice runs V = 0 from the identity and writes the
  //           segment's dk x dk transition M_p to Mws slot p-1.
  //   mode 2: segments 1 .. n_segs-1 from their start states S_p in Sst slot
  //           p-1, with outputs; the last segment writes S_T.
  //   mode 3: the state pass of the corrected schedule: as mode 1, but for
  //           segments 1 .. n_segs-1 (B_p, M_p in slot p-1), and with
  //           outputs: the slices write each segment's zero-start output o^0
  //           into o, the transition slice its outputs
  //           qhat_i = scale qn_i M_{p,i}^T q_i (the start state's share of
  //           o_i is then qhat_i^T S_p, added by gdn_segment_correct_kernel)
  //           into qhat [tokens][H][dk].  It runs without the output gate and
  //           the loop residual, which the correction applies.
  int mode, n_segs, seg_tok, seg0_tok;
  const int32_t* order;  // mode 0, varlen: sequences longest first (block order), or null
  float* Bws;          // [n_seq][n_part][H][dk][dv], n_part = n_segs-2 (mode 1) or n_segs-1 (mode 3)
  float* Mws;          // [n_seq][n_part][H][dk][dk]
  float* Sst;          // [n_seq][n_segs-1][H][dk][dv]
  __nv_bfloat16* qhat; // mode 3: [total_tokens][H][dk]
};

// Per-chunk gate vectors (one buffer).
struct Gates {
  float* g2;     // prefix sum of log2 a (log2 gamma)
  float* gamma;  // exp(g)
  float* b;      // write strength (0 past the sequence end)
  float* bg;     // b * gamma
  float* r;      // gamma_C / gamma = exp(g_C - g)
  float* e;      // 2^(g2_i - m), m = (g2_0 + g2_{C-1}) / 2 (row factor of D)
  float* f;      // 2^(m - g2_j) (column factor of D)
  float* flag;   // [0]: 1 when |g2_0 - g2_{C-1}| < 64, so that e_i f_j = D_ij in range
  // With the q/k L2 norm the tiles stay as loaded and the state team folds the
  // inverse row norms into the factors that meet them: r, bg and f take
  // 1/|k_j| (f becomes 1/|k_j| alone when flag is 0), and qn, gq take 1/|q_i|.
  float* gq;     // gamma_i qn_i (output factor of Sigma^T Q^T)
  float* kn;     // 1 / |k_i|
  float* qn;     // output row factor: sigmoid(gate_i) (1 without the gate), times 1/|q_i|
};

__device__ __forceinline__ Gates gates_at(uint8_t* sm, int buf) {
  float* base = reinterpret_cast<float*>(sm + OFF_GATE + buf * GATE_BYTES);
  return Gates{base,       base + 64,  base + 128, base + 192, base + 256, base + 320,
               base + 384, base + 448, base + 512, base + 576, base + 640};
}

// Named barrier of one warpgroup (the warp is reconverged first: the barrier is
// warp-aligned and the bounded waits exit lane by lane).
template <int ID>
__device__ __forceinline__ void wg_sync() {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(TEAM) : "memory");
}

// Team barrier that also ORs a predicate over its 256 threads
// (bar.red.or): every thread gets the same answer, even when the abort flag is
// set by the other warpgroup while the threads are reading it.
template <int ID>
__device__ __forceinline__ bool wg_sync_or(bool pred) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(ID), "n"(TEAM)
      : "memory");
  return r != 0;
}

// All threads of a warpgroup wait on `bar`; the outcome (abort flag seen by any
// thread) is made uniform so that no thread leaves the schedule alone.
template <int ID>
__device__ __forceinline__ bool wg_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                        unsigned* status) {
  mbar_wait_bounded(bar, parity, abort, status);
  return !wg_sync_or<ID>(*abort != 0);
}

// K-major, 128-byte swizzled operand: rows of 128 bytes, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return smem_desc(saddr, 16, 1024); }
// MN-major, 128-byte swizzled operand: 64 contiguous MN elements per 128-byte row,
// rows along K 128 B apart (8-row atoms 1024 B apart), next 64 MN elements `lbo` bytes on.
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr, uint32_t lbo) {
  return smem_desc(saddr, lbo, 1024);
}

// Normalise one 128-element bf16 row of a [K0|Q0|K1|Q1] stage tile in place:
// x / sqrt(sum x^2 + eps) in fp32, rounded to bf16.
// Inverse L2 norms of the chunk's 64 K rows and 64 Q rows (one stage of K/Q
// tiles, as loaded) for the 256 threads of a team, two threads per row, each
// summing the squares of one 64-column slab; the factors are folded into the
// chunk's gate vectors (see struct Gates).  Every thread of the team calls it
// (warp shuffles); it reads shared memory only, so after a failed wait it just
// produces values that the abort discards.
__device__ __forceinline__ void fold_qk_norms(const uint8_t* kq, const Gates& G, int t) {
  const int row = t >> 1, slab = t & 1;            // rows 0-63: K, 64-127: Q
  const int r = row & 63;
  const uint32_t base = (row < C ? 0u : 8192u) + slab * 16384u;
  uint4 v[8];                                      // all loads first, then the sums
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = *reinterpret_cast<const uint4*>(kq + base + sw128_offset(r, c * 8));
  float ss[4] = {0.f, 0.f, 0.f, 0.f};              // four independent partial sums
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bf16_lo(w[e]), hi = bf16_hi(w[e]);
      ss[e] = fmaf(lo, lo, ss[e]);
      ss[e] = fmaf(hi, hi, ss[e]);
    }
  }
  float sum = (ss[0] + ss[1]) + (ss[2] + ss[3]);
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  const float inv = rsqrtf(sum + kQkNormEps);
  if (slab == 0) {
    if (row < C) {
      G.kn[r] = inv;
      G.r[r] *= inv;
      G.bg[r] *= inv;
      G.f[r] = (G.flag[0] != 0.f ? G.f[r] : 1.f) * inv;
    } else {
      const float qs = G.qn[r] * inv;
      G.qn[r] = qs;
      G.gq[r] = G.gamma[r] * qs;
    }
  }
}

// Writes 32 fp32 values as bf16 into columns [col0, col0 + 32) of one row of a
// 128-byte-swizzled tile with 128-byte rows (four 16-byte chunks).
__device__ __forceinline__ void store_row32_bf16(uint8_t* tile, int row, int col0, const float (&x)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 o;
    o.x = pack_bf16x2(x[c * 8 + 0], x[c * 8 + 1]);
    o.y = pack_bf16x2(x[c * 8 + 2], x[c * 8 + 3]);
    o.z = pack_bf16x2(x[c * 8 + 4], x[c * 8 + 5]);
    o.w = pack_bf16x2(x[c * 8 + 6], x[c * 8 + 7]);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, col0 + c * 8)) = o;
  }
}

// 2^x with the hardware base-2 exponential (relative error about 2^-22;
// results below 2^-126 flush to zero).  Every decay factor of the chunk is
// 2^(g2_i - g2_j) with g2 = log2 gamma.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warp-level m16n8k8 tf32 MMA (fp32 accumulate) for the 16 x 16 blocks of the
// solve, with each operand split into a tf32 high part and a tf32 remainder:
// a b ~= ah bh + ah bl + al bh, which keeps the products close to fp32.  The
// three partial products go to separate accumulators (independent chains).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Fragments of one compact 16 x 16 block (g = lane / 4, q = lane % 4):
// as the A operand (two k-steps of 16 x 8) or as the B operand (two k-steps
// x two n-tiles of 8 x 8).
__device__ __forceinline__ void frag_a(float (&a)[2][4], const float* blkp, int g, int q) {
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    a[ks][0] = blkp[g * BLK_LD + ks * 8 + q];
    a[ks][1] = blkp[(g + 8) * BLK_LD + ks * 8 + q];
    a[ks][2] = blkp[g * BLK_LD + ks * 8 + q + 4];
    a[ks][3] = blkp[(g + 8) * BLK_LD + ks * 8 + q + 4];
  }
}
// B-operand fragments of one 8-column n-tile `nt` of a compact block (two
// k-steps of 8 x 8).
__device__ __forceinline__ void frag_b(float (&b)[2][2], const float* blkp, int nt, int g, int q) {
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    b[ks][0] = blkp[(ks * 8 + q) * BLK_LD + nt * 8 + g];
    b[ks][1] = blkp[(ks * 8 + q + 4) * BLK_LD + nt * 8 + g];
  }
}
// acc[term] += A B for one block pair (K = 16), one n-tile
__device__ __forceinline__ void mma_blk(float (&acc)[3][4], const float (&a)[2][4], const float (&b)[2][2]) {
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
    for (int e = 0; e < 4; ++e) split_tf32(a[ks][e], ah[e], al[e]);
    split_tf32(b[ks][0], bh[0], bl[0]);
    split_tf32(b[ks][1], bh[1], bl[1]);
    mma_tf32(acc[0], ah, bh);
    mma_tf32(acc[1], ah, bl);
    mma_tf32(acc[2], al, bh);
  }
}
__device__ __forceinline__ void acc_zero(float (&acc)[3][4]) {
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
}
// Sums the three partial products, times `sign`, into the accumulator layout
// (res = rows g, g, g+8, g+8 x columns nt*8 + 2q, +1, 2q, +1).
__device__ __forceinline__ void acc_sum(float (&res)[4], const float (&acc)[3][4], float sign) {
#pragma unroll
  for (int e = 0; e < 4; ++e) res[e] = sign * (acc[0][e] + (acc[1][e] + acc[2][e]));
}
__device__ __forceinline__ void store_res(float* blkp, const float (&res)[4], int nt, int g, int q) {
  *reinterpret_cast<float2*>(blkp + g * BLK_LD + nt * 8 + 2 * q) = make_float2(res[0], res[1]);
  *reinterpret_cast<float2*>(blkp + (g + 8) * BLK_LD + nt * 8 + 2 * q) = make_float2(res[2], res[3]);
}
// n-tile nt of T block (a, b) from the accumulator layout into the bf16
// operands T1 = T diag(b gamma) and T2 = T diag(b).
__device__ __forceinline__ void store_res_t12(uint8_t* sm, const Gates& G, int a, int b,
                                              const float (&res)[4], int nt, int g, int q) {
  const int col = b * 16 + nt * 8 + 2 * q;
  const float2 bg = *reinterpret_cast<const float2*>(G.bg + col);
  const float2 bb = *reinterpret_cast<const float2*>(G.b + col);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = a * 16 + g + 8 * h;
    const float x0 = res[2 * h], x1 = res[2 * h + 1];
    *reinterpret_cast<uint32_t*>(sm + OFF_T1 + sw128_offset(row, col)) = pack_bf16x2(x0 * bg.x, x1 * bg.y);
    *reinterpret_cast<uint32_t*>(sm + OFF_T2 + sw128_offset(row, col)) = pack_bf16x2(x0 * bb.x, x1 * bb.y);
  }
}

// Gate inputs of one token (threads 0-63 of the state warpgroup): a, b and,
// with the looped-block epilogue (EPI), the output gate sigmoid(gate) (1
// without one), or a = 1, b = 0 past the sequence end.  Issued well before
// they are used so the global-memory latency is hidden behind a chunk.
template <bool EPI>
__device__ __forceinline__ void load_gate_inputs(const Params& p, int tok0, int valid, int h, int t,
                                                 float& a_in, float& bb, float& og) {
  a_in = 1.f;
  bb = 0.f;
  og = 1.f;
  if (t < valid) {
    const size_t ti = (size_t)(tok0 + t) * p.H + h;
    a_in = __ldg(p.a + ti);
    bb = __ldg(p.b + ti);
    if (EPI && p.gate) og = 1.f / (1.f + __expf(-__ldg(p.gate + ti)));
  }
}

// Gate vectors of one chunk (all 128 threads of a warpgroup call this; threads
// 0-63 own one token each).  Rows past the sequence end get a = 1 and b = 0.
template <int BAR>
__device__ __forceinline__ void compute_gates(Gates G, float* s_carry, int valid, int t, float a_in,
                                              float bb, float og) {
  const int lane = t & 31;
  float la = 0.f;
  if (t < C) {
    la = (t < valid) ? log2f(a_in) : 0.f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, la, off);
      if (lane >= off) la += y;
    }
    if (t == 31) *s_carry = la;
    G.b[t] = bb;
  }
  wg_sync<BAR>();
  if (t < C) {
    if (t >= 32) la += *s_carry;
    G.g2[t] = la;
  }
  wg_sync<BAR>();
  if (t < C) {
    const float g0 = G.g2[0], gl = G.g2[C - 1];
    const float mid = 0.5f * (g0 + gl);
    const float gam = ex2_approx(la);
    G.gamma[t] = gam;
    G.qn[t] = og;
    G.gq[t] = gam * og;
    G.bg[t] = bb * gam;
    G.r[t] = ex2_approx(gl - la);
    G.e[t] = ex2_approx(la - mid);
    G.f[t] = ex2_approx(mid - la);
    if (t == 0) G.flag[0] = (fabsf(g0 - gl) < 64.f) ? 1.f : 0.f;
  }
}

// x <- L^{-1} x for the unit lower 16 x 16 diagonal block L = I + A_LL of A
// (compact block `ad`), one right-hand side per thread.  Rows of A are read 4
// entries at a time; A's entries on and above its diagonal are stored as zeros,
// so whole 4-vectors can be used.
__device__ __forceinline__ void fwd_subst16(const float* ad, float (&x)[16]) {
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < i; m += 4) {
      const float4 a4 = *reinterpret_cast<const float4*>(ad + i * BLK_LD + m);
      acc[0] = fmaf(a4.x, x[m], acc[0]);
      acc[1] = fmaf(a4.y, x[m + 1], acc[1]);
      acc[2] = fmaf(a4.z, x[m + 2], acc[2]);
      acc[3] = fmaf(a4.w, x[m + 3], acc[3]);
    }
    x[i] -= (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
}

// T = (I + A)^{-1} for the strictly lower 64 x 64 matrix A, both in compact
// block form, by recursive doubling of the 2 x 2 block inverse
//     [[L1, 0], [M, L2]]^{-1} = [[L1^-1, 0], [-(L2^-1 M) L1^-1, L2^-1]].
// Forward substitution inside the 16 x 16 diagonal blocks gives, in one pass,
// the four T_aa = L_a^-1 and Z_{a+1,a} = L_{a+1}^-1 A_{a+1,a} for a = 0, 2;
// then T_{a+1,a} = -Z_{a+1,a} T_aa, and the 32 x 32 block below the diagonal
// as Y = A_21 T_top, T_21 = -T_bot Y (warp-level tf32 MMAs, 3xTF32, one
// 8-column n-tile per warp).  Every T block is also written, rounded to bf16
// and column-scaled, into the T1 and T2 operand tiles (their upper block
// triangle is zero from the start).  All 256 threads of the prep team call it.
__device__ __forceinline__ void solve_t(uint8_t* sm, const Gates& G, const float* s_A, float* s_T,
                                        int t) {
  const int warp = t >> 5, lane = t & 31;
  const int g = lane >> 2, q = lane & 3;
  if (t < 96) {
    // threads 0-63: T_aa column c (a = t / 16); 64-79: Z_10 column c; 80-95: Z_32 column c
    const int c = t & 15;
    const int L = (t < 64) ? (t >> 4) : ((t < 80) ? 1 : 3);
    const bool rhs_a = (t >= 64);
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      x[i] = rhs_a ? s_A[blk(L, L - 1) + i * BLK_LD + c] : ((i == c) ? 1.f : 0.f);
    fwd_subst16(s_A + blk(L, L), x);
    float* out = s_T + (rhs_a ? blk(L, L - 1) : blk(L, L));
#pragma unroll
    for (int i = 0; i < 16; ++i) out[i * BLK_LD + c] = x[i];
  }
  wg_sync<BAR_PREP>();
  {
    // warps 0-3: T_{a+1,a} = -Z_{a+1,a} T_aa (a = 0, 2), n-tile warp % 2, over Z in place;
    // warps 4-7 meanwhile: the diagonal blocks into T1 and T2 (one row half per thread)
    const int a = (warp >> 1) * 2, nt = warp & 1;
    float fa[2][4], fb[2][2], acc[3][4], res[4];
    if (warp < 4) {
      frag_a(fa, s_T + blk(a + 1, a), g, q);
      frag_b(fb, s_T + blk(a, a), nt, g, q);
    } else {
      const int u = t - 128;                 // 0..127
      const int ad = u >> 5, r = (u >> 1) & 15, half = u & 1;
      const float* src = s_T + blk(ad, ad) + r * BLK_LD + half * 8;
      const float4 x0 = *reinterpret_cast<const float4*>(src);
      const float4 x1 = *reinterpret_cast<const float4*>(src + 4);
      const int col = ad * 16 + half * 8, row = ad * 16 + r;
      const float4 bg0 = *reinterpret_cast<const float4*>(G.bg + col);
      const float4 bg1 = *reinterpret_cast<const float4*>(G.bg + col + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(G.b + col);
      const float4 b1 = *reinterpret_cast<const float4*>(G.b + col + 4);
      uint4 o1, o2;
      o1.x = pack_bf16x2(x0.x * bg0.x, x0.y * bg0.y);
      o1.y = pack_bf16x2(x0.z * bg0.z, x0.w * bg0.w);
      o1.z = pack_bf16x2(x1.x * bg1.x, x1.y * bg1.y);
      o1.w = pack_bf16x2(x1.z * bg1.z, x1.w * bg1.w);
      o2.x = pack_bf16x2(x0.x * b0.x, x0.y * b0.y);
      o2.y = pack_bf16x2(x0.z * b0.z, x0.w * b0.w);
      o2.z = pack_bf16x2(x1.x * b1.x, x1.y * b1.y);
      o2.w = pack_bf16x2(x1.z * b1.z, x1.w * b1.w);
      *reinterpret_cast<uint4*>(sm + OFF_T1 + sw128_offset(row, col)) = o1;
      *reinterpret_cast<uint4*>(sm + OFF_T2 + sw128_offset(row, col)) = o2;
    }
    wg_sync<BAR_PREP>();                     // both n-tile warps have read Z before it is replaced
    if (warp < 4) {
      acc_zero(acc);
      mma_blk(acc, fa, fb);
      acc_sum(res, acc, -1.f);
      store_res(s_T + blk(a + 1, a), res, nt, g, q);
      store_res_t12(sm, G, a + 1, a, res, nt, g, q);
    }
  }
  wg_sync<BAR_PREP>();
  // Y_{a,b} = sum_{k=b}^{1} A_{a,k} T_{k,b}  (a = 2, 3; b = 0, 1), n-tile warp % 2, into block (a, b)
  const int bk = warp >> 1, nt = warp & 1;
  const int a2 = 2 + (bk >> 1), b2 = bk & 1;
  {
    float fa[2][4], fb[2][2], acc[3][4], res[4];
    acc_zero(acc);
    frag_a(fa, s_A + blk(a2, 1), g, q);
    frag_b(fb, s_T + blk(1, b2), nt, g, q);
    mma_blk(acc, fa, fb);
    if (b2 == 0) {
      frag_a(fa, s_A + blk(a2, 0), g, q);
      frag_b(fb, s_T + blk(0, 0), nt, g, q);
      mma_blk(acc, fa, fb);
    }
    acc_sum(res, acc, 1.f);
    store_res(s_T + blk(a2, b2), res, nt, g, q);
  }
  wg_sync<BAR_PREP>();
  // T_{a,b} = -sum_{m=2}^{a} T_{a,m} Y_{m,b}
  {
    float fa0[2][4], fb0[2][2], fa1[2][4], fb1[2][2], acc[3][4], res[4];
    frag_a(fa0, s_T + blk(a2, a2), g, q);
    frag_b(fb0, s_T + blk(a2, b2), nt, g, q);
    if (a2 == 3) {
      frag_a(fa1, s_T + blk(3, 2), g, q);
      frag_b(fb1, s_T + blk(2, b2), nt, g, q);
    }
    wg_sync<BAR_PREP>();                   // every Y is read before any is replaced
    acc_zero(acc);
    mma_blk(acc, fa0, fb0);
    if (a2 == 3) mma_blk(acc, fa1, fb1);
    acc_sum(res, acc, -1.f);
    store_res(s_T + blk(a2, b2), res, nt, g, q);
    store_res_t12(sm, G, a2, b2, res, nt, g, q);
  }
}

// Half hf (dk columns 64 hf .. 64 hf + 63) of Sigma^T row j (fp32, in tensor
// memory) -> bf16 operand tile (slab hf) for the next chunk; the tensor-memory
// copy is scaled by `decay` (gamma_C of the next chunk) so that the next carry
// MMA accumulates onto gamma_C Sigma.  With `st_out`, the unscaled fp32 row is
// also written to S_T (rows dk, row stride `ld`).
__device__ __forceinline__ void refresh_state(uint32_t taddr, uint8_t* sig, int j, int hf, float decay,
                                              bool scale_tmem, float* st_out, int ld) {
#pragma unroll 1
  for (int piece = 0; piece < 2; ++piece) {
    float x[32];
    const uint32_t col = hf * 64 + piece * 32;
    tmem_ld32(taddr + col, x);
    store_row32_bf16(sig + hf * 16384, j, piece * 32, x);
    if (st_out) {
#pragma unroll
      for (int e = 0; e < 32; ++e) st_out[(size_t)(col + e) * ld] = x[e];
    }
    if (scale_tmem) {
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= decay;
      tmem_st32(taddr + col, x);
    }
  }
  tmem_wait_st();
}

// TMA loads of one chunk: K and Q into stage s, or the V slice.
__device__ __forceinline__ void load_kq(uint8_t* sm, uint64_t* bar, const CUtensorMap* tq,
                                        const CUtensorMap* tk, int s, int h, int tok0) {
  uint8_t* kq = sm + OFF_KQ + s * KQ_BYTES;
  mbar_arrive_expect_tx(bar, KQ_BYTES);
  tma_load_3d(kq + 0, tk, bar, 0, h, tok0);
  tma_load_3d(kq + 16384, tk, bar, 64, h, tok0);
  tma_load_3d(kq + 8192, tq, bar, 0, h, tok0);
  tma_load_3d(kq + 24576, tq, bar, 64, h, tok0);
}
__device__ __forceinline__ void load_v(uint8_t* sm, uint64_t* bar, const CUtensorMap* tv, int col0,
                                       int h, int tok0) {
  mbar_arrive_expect_tx(bar, V_BYTES);
  tma_load_3d(sm + OFF_V, tv, bar, col0, h, tok0);
  tma_load_3d(sm + OFF_V + 8192, tv, bar, col0 + 64, h, tok0);
}
// EPI: the looped-block epilogue (output gate, loop residual) is compiled in;
// the plain mixer call runs the instance without it.
template <bool EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gdn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {   // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_status(p.status, GDN_ERR_CUDA);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  // loads issued so far: K/Q per stage, V (read back to drain in-flight copies on exit)
  volatile int* s_issued = reinterpret_cast<volatile int*>(sm + OFF_MISC + 16);

  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);   // warp-uniform by construction
  // segmented schedule: the combine kernel may be launched now (it waits for
  // this grid before it reads anything)
  if (p.mode == 1 || p.mode == 3) griddep_launch_dependents();

  // work unit: (sequence or segment, head, dv slice)
  int slice, h, seq, part;
  bool partial = false;   // a segment run from a zero state or the identity
  const bool state_pass = (p.mode == 1 || p.mode == 3);
  const int n_part = (p.mode == 3) ? p.n_segs - 1 : p.n_segs - 2;   // segments with B, M
  {
    int bid = (int)blockIdx.x;
    int slices_here = p.n_slices;
    int units_per_seq = 1, first_part = 0;
    if (state_pass) {
      const int n_first = p.n_seq * p.H * p.n_slices;   // segment 0 of every chain, run in full
      if (bid >= n_first) {
        bid -= n_first;
        partial = true;
        slices_here = p.n_slices + 1;
        units_per_seq = n_part;
        first_part = 1;
      }
    } else if (p.mode == 2) {
      units_per_seq = p.n_segs - 1;
      first_part = 1;
    }
    slice = bid % slices_here;
    const int chain = bid / slices_here;
    h = chain % p.H;
    const int unit = chain / p.H;
    seq = unit / units_per_seq;
    part = first_part + unit % units_per_seq;
    if (p.order) seq = __ldg(p.order + seq);   // longest sequences in the first blocks
  }
  const bool ident = partial && slice == p.n_slices;   // transition slice: V = 0, S0 = I
  // outputs: whole segments, and every segment of the corrected state pass
  // (zero-start outputs, or qhat from the transition slice); the loop residual
  // only where the output is final
  const bool outputs = !partial || p.mode == 3;
  const bool residual = EPI && (p.h_prev != nullptr) && !partial;
  int seq_start, seq_end;
  if (p.cu_seqlens) {
    seq_start = p.cu_seqlens[seq];
    seq_end = p.cu_seqlens[seq + 1];
  } else {
    seq_start = seq * p.seq_len;
    seq_end = seq_start + p.seq_len;
    if (p.mode != 0) {
      seq_start += (part == 0) ? 0 : p.seg0_tok + (part - 1) * p.seg_tok;
      seq_end = min(seq_end, seq_start + (part == 0 ? p.seg0_tok : p.seg_tok));
    }
  }
  {
    // offsets outside [0, total_tokens] or decreasing: clamp, and report
    const int s0 = min(max(seq_start, 0), p.total_tokens);
    const int s1 = min(max(seq_end, s0), p.total_tokens);
    if ((s0 != seq_start || s1 != seq_end) && tid == 0) record_status(p.status, GDN_ERR_INVALID);
    seq_start = s0;
    seq_end = s1;
  }
  const int len = seq_end - seq_start;
  const int n_chunks = (len + C - 1) / C;
  const int H = p.H, dv = p.dv;
  const int col0 = ident ? 0 : slice * DVS;

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], 1);
    *s_abort = 0;
    s_issued[0] = s_issued[1] = s_issued[2] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = smem_u32(sm);
  if (tid == 0 && n_chunks > 0) {
    // first loads: K/Q of chunks 0 and 1, V of chunk 0
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    load_kq(sm, &bars[B_KQ_FULL + 0], &tm_q, &tm_k, 0, h, seq_start);
    s_issued[0] = 1;
    if (n_chunks > 1) {
      load_kq(sm, &bars[B_KQ_FULL + 1], &tm_q, &tm_k, 1, h, seq_start + C);
      s_issued[1] = 1;
    }
    if (!ident) {
      load_v(sm, &bars[B_V_FULL], &tm_v, col0, h, seq_start);
      s_issued[2] = 1;
    }
  }

  if (warp < 8) {
    // ================================================================ prep team
    const int t = tid;                       // 0..255
    const int lane = t & 31;
    const int hf = t >> 7;                   // column half of a tensor-memory row
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float* s_A = reinterpret_cast<float*>(sm + OFF_A);
    float* s_T = reinterpret_cast<float*>(sm + OFF_TS);
    {
      // the upper block triangle of T1 and T2 stays zero for the whole sequence
      uint4* z = reinterpret_cast<uint4*>(sm + OFF_T1);
      for (int u = t; u < 2 * 8192 / 16; u += TEAM) z[u] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t pphase = 0;
    const bool l2n = (p.flags & GDN_QK_L2NORM) != 0;
    bool ok = true;
#pragma unroll 1
    for (int c = 0; c < n_chunks && ok; ++c) {
      const int s = c & 1;
      const int tok0 = seq_start + c * C;
      const Gates G = gates_at(sm, c % 3);
      const uint32_t kq_a = sbase + OFF_KQ + s * KQ_BYTES;

      // ---- G of chunk c and its gate vectors (both from the state team, the
      // gates with the q/k norms folded in), and the P and U buffers s (free
      // once chunk c-2 is finished): each thread waits on the three barriers,
      // then one team barrier makes the outcome uniform
      {
        bool okw = mbar_wait_bounded(&bars[B_G_MMA + s], (c >> 1) & 1, s_abort, p.status);
        okw = okw && mbar_wait_bounded(&bars[B_GATES + c % 3], (c / 3) & 1, s_abort, p.status);
        if (c >= 2)
          okw = okw && mbar_wait_bounded(&bars[B_CHUNK_DONE + s], ((c >> 1) - 1) & 1, s_abort, p.status);
        if (wg_sync_or<BAR_PREP>(!okw || *s_abort != 0)) break;   // a failed wait set the abort flag
      }
      tc_fence_after();
      {
        // A = strict_lower(diag(b) (D o K K^T)) (rows 0-63, fp32, compact blocks) and
        // P = tril(D o Q K^T) (rows 64-127, bf16 operand), D_ij = 2^(g2_i - g2_j),
        // taken as e_i f_j when the chunk's decay range allows (no exponential per
        // entry), else one exponential per entry.  Thread t owns columns
        // 32 hf .. 32 hf + 31 of row i of its half; rows 0-31 (warps 0, 2, 4, 6)
        // have only zeros in columns 32-63.
        const int tq = t & 127;
        const int i = tq & 63;
        const int cb = hf * 32;                         // first column of this thread
        const bool zero_half = (hf == 1) && ((warp & 1) == 0);
        // row factor: b_i (A rows) or the output row factor qn_i (P rows: the
        // output gate and 1/|q_i|), times 1/|k_i| on A rows with the norm; the
        // column factor f_j carries 1/|k_j| (and is 1/|k_j| alone on the
        // exponential path)
        const float sc = (tq < C) ? (l2n ? G.b[i] * G.kn[i] : G.b[i]) : ((EPI || l2n) ? G.qn[i] : 1.f);
        const int lim = (tq < C) ? i : i + 1;           // columns j < lim are kept
        float gr[32];
        if (zero_half) {
#pragma unroll
          for (int e = 0; e < 32; ++e) gr[e] = 0.f;
        } else {
          tmem_ld32(tmem + lane_off + col_gw(c) + cb, gr);
          if (G.flag[0] != 0.f) {
            const float sce = sc * G.e[i];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 f4 = *reinterpret_cast<const float4*>(G.f + cb + 4 * j4);
              const float fv[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int jj = cb + 4 * j4 + e;
                gr[4 * j4 + e] = (jj < lim) ? (gr[4 * j4 + e] * fv[e]) * sce : 0.f;
              }
            }
          } else {
            const float gi = G.g2[i];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 gj = *reinterpret_cast<const float4*>(G.g2 + cb + 4 * j4);
              const float gjv[4] = {gj.x, gj.y, gj.z, gj.w};
              const float4 f4 = l2n ? *reinterpret_cast<const float4*>(G.f + cb + 4 * j4)
                                    : make_float4(1.f, 1.f, 1.f, 1.f);
              const float fv[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int jj = cb + 4 * j4 + e;
                const float d = ex2_approx(gi - gjv[e]);
                gr[4 * j4 + e] = (jj < lim) ? (sc * gr[4 * j4 + e]) * (d * fv[e]) : 0.f;
              }
            }
          }
        }
        if (tq < C) {
          const int I = i >> 4;
          float* arow = s_A + (i & 15) * BLK_LD;
#pragma unroll
          for (int bl = 0; bl < 2; ++bl) {
            const int bj = 2 * hf + bl;
            if (bj <= I) {
              float4* dst = reinterpret_cast<float4*>(arow + blk(I, bj));
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_float4(gr[16 * bl + 4 * k], gr[16 * bl + 4 * k + 1], gr[16 * bl + 4 * k + 2],
                                     gr[16 * bl + 4 * k + 3]);
            }
          }
        } else {
          store_row32_bf16(sm + OFF_P + s * 8192, i, cb, gr);
        }
      }
      tc_fence_before();
      wg_sync<BAR_PREP>();

      // ---- T = (I + A)^{-1}, written as T1 = T diag(b gamma), T2 = T diag(b) (bf16)
      solve_t(sm, G, s_A, s_T, t);
      fence_proxy_async_smem();
      wg_sync<BAR_PREP>();

      // ---- U~^T = V^T T2^T (into U buffer s) and W^T = K^T T1^T (M = 128, N = 64, K = 64 tokens).
      // Warp 0 issues them and alone takes the waits they need (V; then the
      // buffer of W^T(c-1), free once the state team has read it), waits for the
      // products and arrives W_READY.  The other warps go straight on to chunk
      // c+1; the team barrier at its top also waits for warp 0, which has seen
      // these products complete by then, so the T1/T2 tiles they overwrite in
      // the next solve are free.  No warp leaves the loop alone: after a failed
      // wait warp 0 only skips work, and the next team barrier sees the abort
      // flag.  Waiting for
      // W_CONSUMED(c-1) in every chunk also keeps W_READY from running two
      // phases ahead of the state team.
      if (warp == 0) {
        // (every wait's outcome is made warp-uniform before the elected lane acts on it)
        bool okw = ident || __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_V_FULL], c & 1, s_abort, p.status));
        tc_fence_after();
        if (okw) {
          const uint32_t v_a = sbase + OFF_V;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
              if (!ident)
                mma_bf16(tmem + COL_U + s * 64, mndesc(v_a + kk * 2048, 8192),
                         kdesc(sbase + OFF_T2 + kk * 32), idesc_bf16(128, 64, 1, 0), kk > 0);
              mma_bf16(tmem + col_gw(c), mndesc(kq_a + kk * 2048, 16384), kdesc(sbase + OFF_T1 + kk * 32),
                       idesc_bf16(128, 64, 1, 0), kk > 0);
            }
            mma_commit(&bars[B_PREP_MMA]);
          }
        }
        __syncwarp();
        if (okw && c >= 1)
          okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_W_CONSUMED], (c - 1) & 1, s_abort, p.status));
        if (okw) okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[B_PREP_MMA], pphase, s_abort, p.status));
        pphase ^= 1;
        if (okw && lane == 0) {
          tc_fence_before();
          mbar_arrive(&bars[B_W_READY]);     // U~^T and W^T of chunk c are in tensor memory
          if (!ident && c + 1 < n_chunks) {  // the V stage is free: load V of chunk c+1
            load_v(sm, &bars[B_V_FULL], &tm_v, col0, h, tok0 + C);
            s_issued[2] = c + 2;
          }
        }
        __syncwarp();
      }
    }
  } else {
    // ================================================================ state team
    const int jt = tid - TEAM;                                // 0..255
    const int j = jt & 127;                                   // dv row owned (tensor-memory lane)
    const int hf = jt >> 7;                                   // column half of the row
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool l2n = (p.flags & GDN_QK_L2NORM) != 0;
    // initial state: s0 (rows dk, row stride ld0), the identity (transition
    // slice) or zero; final state to st (row stride ldT) or nowhere
    const size_t state_base = ((size_t)seq * H + h) * DK * (size_t)dv + col0 + j;
    const float* s0 = nullptr;
    float* st = nullptr;
    size_t ldT = dv;
    if (p.mode == 0) {
      s0 = p.S0 ? p.S0 + state_base : nullptr;
      st = p.S_T ? p.S_T + state_base : nullptr;
    } else if (state_pass && !partial) {   // segment 0: S_1 to start-state slot 0
      s0 = p.S0 ? p.S0 + state_base : nullptr;
      st = p.Sst + ((size_t)seq * (p.n_segs - 1) * H + h) * DK * (size_t)dv + col0 + j;
    } else if (state_pass) {
      const size_t u = (size_t)seq * n_part + (part - 1);
      if (ident) {
        st = p.Mws + (u * H + h) * DK * DK + j;
        ldT = DK;
      } else {
        st = p.Bws + (u * H + h) * DK * (size_t)dv + col0 + j;
      }
    } else {
      s0 = p.Sst + (((size_t)seq * (p.n_segs - 1) + (part - 1)) * H + h) * DK * (size_t)dv + col0 + j;
      if (part == p.n_segs - 1 && p.S_T) st = p.S_T + state_base;
    }
    uint32_t sphase = 0;
    bool ok = true;

    if (p.flags & GDN_TEST_WAIT_TIMEOUT) {
      // test hook: a wait that nothing ends runs out, records GDN_ERR_TIMEOUT
      // and sets the abort flag, which ends every other wait of the block
      if (jt == 0) mbar_wait_bounded(&bars[B_NEVER], 0, s_abort, p.status);
      ok = !wg_sync_or<BAR_STATE>(*s_abort != 0);
    }
    float* s_carry = reinterpret_cast<float*>(sm + OFF_MISC + 8);
    // gate vectors of chunks 0 and 1 (later ones are built two chunks ahead,
    // while the products of each chunk run); a_in, b_in hold the inputs of the
    // next chunk to build
    float a_in, b_in, og_in;
    auto gates_of = [&](int c) {
      compute_gates<BAR_STATE>(gates_at(sm, c % 3), s_carry, min(C, seq_end - (seq_start + c * C)), jt,
                               a_in, b_in, og_in);
      if (c + 1 < n_chunks)
        load_gate_inputs<EPI>(p, seq_start + (c + 1) * C, min(C, seq_end - (seq_start + (c + 1) * C)), h,
                              jt, a_in, b_in, og_in);
      wg_sync<BAR_STATE>();
    };
    // Hands chunk c2 to the prep team once its K, Q tiles have landed: with the
    // norm flag the inverse row norms are folded into its gate vectors (the
    // tiles stay as loaded), the gates are released, and warp 8 issues
    // G = [K; Q] K^T (M = 128, N = 64, K = dk) into tensor-memory buffer
    // c2 % 2, whose last content, W^T of chunk c2-2, this team has read.
    // Returns false (uniformly) if the wait gave up.
    auto release_chunk = [&](int c2) -> bool {
      const int s2 = c2 & 1;
      if (!wg_wait<BAR_STATE>(&bars[B_KQ_FULL + s2], (c2 >> 1) & 1, s_abort, p.status)) return false;
      if (l2n) {
        fold_qk_norms(sm + OFF_KQ + s2 * KQ_BYTES, gates_at(sm, c2 % 3), jt);
        wg_sync<BAR_STATE>();
      }
      if (jt == 0) mbar_arrive(&bars[B_GATES + c2 % 3]);
      if (warp == 8) {
        tc_fence_after();
        if (elect_one()) {
          const uint32_t kq2 = sbase + OFF_KQ + s2 * KQ_BYTES;
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16(tmem + col_gw(c2), kdesc(kq2 + off), kdesc(kq2 + off), idesc_bf16(128, 64, 0, 0),
                     kk > 0);
          }
          mma_commit(&bars[B_G_MMA + s2]);
        }
        __syncwarp();
      }
      return true;
    };
    if (ok && n_chunks > 0) {
      load_gate_inputs<EPI>(p, seq_start, min(C, len), h, jt, a_in, b_in, og_in);
      gates_of(0);
      if (n_chunks > 1) gates_of(1);
#pragma unroll 1
      for (int c2 = 0; c2 < min(2, n_chunks) && ok; ++c2) ok = release_chunk(c2);
    }

    // initial state: tensor memory holds gamma_C(0) * S0, the bf16 operand holds S0
    // (this thread: dk columns 64 hf .. 64 hf + 63 of row j).  The output pass
    // may have started before the kernels that write its start states have
    // finished: everything above ran meanwhile, the start state waits for them.
    if (p.mode == 2) griddep_wait();
    const float decay0 = (n_chunks > 0) ? gates_at(sm, 0).gamma[C - 1] : 1.f;
    {
#pragma unroll 1
      for (int piece = 2 * hf; piece < 2 * hf + 2; ++piece) {
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          x[e] = ident ? ((piece * 32 + e == j) ? 1.f : 0.f)
                       : (s0 ? __ldg(s0 + (size_t)(piece * 32 + e) * dv) : 0.f);
        uint8_t* slab = sm + OFF_SIG + (piece >> 1) * 16384;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint4 o;
          o.x = pack_bf16x2(x[cc * 8 + 0], x[cc * 8 + 1]);
          o.y = pack_bf16x2(x[cc * 8 + 2], x[cc * 8 + 3]);
          o.z = pack_bf16x2(x[cc * 8 + 4], x[cc * 8 + 5]);
          o.w = pack_bf16x2(x[cc * 8 + 6], x[cc * 8 + 7]);
          *reinterpret_cast<uint4*>(slab + sw128_offset(j, (piece & 1) * 32 + cc * 8)) = o;
        }
        if (n_chunks == 0 && st) {
#pragma unroll
          for (int e = 0; e < 32; ++e) st[(size_t)(piece * 32 + e) * ldT] = x[e];
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= decay0;
        tmem_st32(tmem + lane_off + COL_S + piece * 32, x);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    wg_sync<BAR_STATE>();

#pragma unroll 1
    for (int c = 0; c < n_chunks && ok; ++c) {
      const int s = c & 1;
      const int tok0 = seq_start + c * C;
      const int valid = min(C, seq_end - tok0);
      const bool last = (c == n_chunks - 1);
      const Gates G = gates_at(sm, c % 3);
      const uint32_t kq_a = sbase + OFF_KQ + s * KQ_BYTES;

      // ---- the rows of h_prev this chunk's epilogue adds (loop residual) into
      // L2, one 128-byte line per thread, so the epilogue's loads do not wait
      // on HBM
      if (outputs && residual && jt < 2 * C) {
        const int i = jt >> 1;
        if (i < valid) {
          const __nv_bfloat16* line = p.h_prev + ((size_t)(tok0 + i) * H + h) * dv + col0 + (jt & 1) * 64;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(line));
        }
      }
      // ---- O_A^T = Sigma^T Q^T (needs no W: it runs while W^T is converted)
      if (!wg_wait<BAR_STATE>(&bars[B_W_READY], c & 1, s_abort, p.status)) break;
      tc_fence_after();
      if (outputs && warp == 8) {
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            mma_bf16(tmem + COL_OA, kdesc(sbase + OFF_SIG + (kk >> 2) * 16384 + (kk & 3) * 32),
                     kdesc(kq_a + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32), idesc_bf16(128, 64, 0, 0),
                     kk > 0);
          mma_commit(&bars[B_OA_MMA]);
        }
        __syncwarp();
      }
      // ---- W^T tile (row d = j, tokens 32 hf ..) out of tensor memory; its buffer
      // is then free for G of chunk c+2
      {
        float wr[32];
        tmem_ld32(tmem + lane_off + col_gw(c) + 32 * hf, wr);
        store_row32_bf16(sm + OFF_WT, j, 32 * hf, wr);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      wg_sync<BAR_STATE>();
      if (jt == 0) mbar_arrive(&bars[B_W_CONSUMED]);
      // ---- U^T -= Sigma^T W^T (onto U~^T in buffer s)
      if (warp == 8) {
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            mma_bf16(tmem + COL_U + s * 64, kdesc(sbase + OFF_SIG + (kk >> 2) * 16384 + (kk & 3) * 32),
                     mndesc(sbase + OFF_WT + kk * 2048, 8192), idesc_bf16(128, 64, 0, 1, /*neg_b=*/1),
                     ident ? (kk > 0) : 1);
          mma_commit(&bars[B_STATE_MMA]);
        }
        __syncwarp();
      }
      if (!wg_wait<BAR_STATE>(&bars[B_STATE_MMA], sphase, s_abort, p.status)) break;
      sphase ^= 1;
      tc_fence_after();

      // ---- U^T row j (tokens 32 hf ..) -> operand tiles U^T and U^T diag(gamma_C / gamma)
      {
        float ur[32];
        tmem_ld32(tmem + lane_off + COL_U + s * 64 + 32 * hf, ur);
        store_row32_bf16(sm + OFF_UT, j, 32 * hf, ur);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 r4 = *reinterpret_cast<const float4*>(G.r + 32 * hf + 4 * e4);
          ur[4 * e4] *= r4.x;
          ur[4 * e4 + 1] *= r4.y;
          ur[4 * e4 + 2] *= r4.z;
          ur[4 * e4 + 3] *= r4.w;
        }
        store_row32_bf16(sm + OFF_UTP, j, 32 * hf, ur);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      wg_sync<BAR_STATE>();

      // ---- O_B^T = U^T P^T (N = 64)  and  Sigma^T += U'^T K (N = dk), K = 64 tokens
      if (warp == 8) {
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) {
            if (outputs)
              mma_bf16(tmem + COL_OB, kdesc(sbase + OFF_UT + kk * 32),
                       kdesc(sbase + OFF_P + s * 8192 + kk * 32), idesc_bf16(128, 64, 0, 0), kk > 0);
            mma_bf16(tmem + COL_S, kdesc(sbase + OFF_UTP + kk * 32), mndesc(kq_a + kk * 2048, 16384),
                     idesc_bf16(128, 128, 0, 1), 1);
          }
          mma_commit(&bars[B_STATE_MMA]);
        }
        __syncwarp();
      }
      // ---- gate vectors of chunk c+2 while the products run (their buffer's
      // previous user, chunk c-1, is finished; they are released with its G)
      if (c + 2 < n_chunks) gates_of(c + 2);
      if (!wg_wait<BAR_STATE>(&bars[B_STATE_MMA], sphase, s_abort, p.status)) break;
      sphase ^= 1;
      tc_fence_after();
      if (jt == 0 && c + 2 < n_chunks) {  // last read of the K, Q stage is done: load chunk c+2
        load_kq(sm, &bars[B_KQ_FULL + s], &tm_q, &tm_k, s, h, tok0 + 2 * C);
        s_issued[s] = (c >> 1) + 2;
      }

      // ---- next chunk's Sigma^T operand (bf16) and pre-decayed fp32 state; S_T at the end
      const float decay = last ? 1.f : gates_at(sm, (c + 1) % 3).gamma[C - 1];   // built by this team
      refresh_state(tmem + lane_off + COL_S, sm + OFF_SIG, j, hf, decay, !last, last ? st : nullptr,
                    (int)ldT);

      // ---- outputs: o[tok0 + i][h][col0 + j] = scale (gamma_i O_A + O_B), staged
      // through shared memory ([64 tok][128 dv] bf16) for 16-byte coalesced stores
      if (outputs) {
        if (!wg_wait<BAR_STATE>(&bars[B_OA_MMA], c & 1, s_abort, p.status)) break;
        tc_fence_after();
        {
          // this thread: dv row j, tokens 32 hf .. 32 hf + 31
          uint8_t* stage = sm + OFF_UTP;
          float oo[32], ob[32];
          tmem_ld32(tmem + lane_off + COL_OA + 32 * hf, oo);
          tmem_ld32(tmem + lane_off + COL_OB + 32 * hf, ob);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 g4 = *reinterpret_cast<const float4*>(((EPI || l2n) ? G.gq : G.gamma) + 32 * hf + 4 * e4);
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              oo[4 * e4 + e] = p.scale * fmaf(oo[4 * e4 + e], gv[e], ob[4 * e4 + e]);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e)
            *reinterpret_cast<__nv_bfloat16*>(stage + (32 * hf + e) * 256 + j * 2) = __float2bfloat16_rn(oo[e]);
        }
        tc_fence_before();
        wg_sync<BAR_STATE>();
        {
          // 16-byte vectors: this thread stores columns col0 + 8 q .. + 7 of rows
          // jt / 16 + 16 k8; with the loop residual it adds rho (.) h_prev of the
          // same elements (read by this thread just before it writes them, so o
          // may be h_prev itself), after the rounding of o, as loop_residual does
          const uint8_t* stage = sm + OFF_UTP;
          const int q = jt & 15;
          // the transition slice of the corrected state pass writes qhat (rows of dk)
          __nv_bfloat16* out = ident ? p.qhat : p.o;
          const int ow = ident ? DK : dv;
          const size_t row0 = ((size_t)tok0 * H + h) * ow + col0 + q * 8;
          const size_t row_stride = (size_t)H * ow;
          if (residual) {
            uint4 hp[4];
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
              const int i = (jt >> 4) + 16 * k8;
              if (i < valid) hp[k8] = *reinterpret_cast<const uint4*>(p.h_prev + row0 + i * row_stride);
            }
            const float4 r0 = __ldg(reinterpret_cast<const float4*>(p.rho + (size_t)h * dv + col0 + q * 8));
            const float4 r1 = __ldg(reinterpret_cast<const float4*>(p.rho + (size_t)h * dv + col0 + q * 8 + 4));
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
              const int i = (jt >> 4) + 16 * k8;
              if (i < valid) {
                const uint4 x = *reinterpret_cast<const uint4*>(stage + i * 256 + q * 16);
                const uint4 y = hp[k8];
                uint4 v;
                v.x = pack_bf16x2(fmaf(r0.x, bf16_lo(y.x), bf16_lo(x.x)), fmaf(r0.y, bf16_hi(y.x), bf16_hi(x.x)));
                v.y = pack_bf16x2(fmaf(r0.z, bf16_lo(y.y), bf16_lo(x.y)), fmaf(r0.w, bf16_hi(y.y), bf16_hi(x.y)));
                v.z = pack_bf16x2(fmaf(r1.x, bf16_lo(y.z), bf16_lo(x.z)), fmaf(r1.y, bf16_hi(y.z), bf16_hi(x.z)));
                v.w = pack_bf16x2(fmaf(r1.z, bf16_lo(y.w), bf16_lo(x.w)), fmaf(r1.w, bf16_hi(y.w), bf16_hi(x.w)));
                __stcs(reinterpret_cast<uint4*>(out + row0 + i * row_stride), v);
              }
            }
          } else {
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
              const int i = (jt >> 4) + 16 * k8;
              if (i < valid) {
                const uint4 v = *reinterpret_cast<const uint4*>(stage + i * 256 + q * 16);
                __stcs(reinterpret_cast<uint4*>(out + row0 + i * row_stride), v);
              }
            }
          }
        }
      }
      fence_proxy_async_smem();
      wg_sync<BAR_STATE>();
      if (jt == 0) mbar_arrive(&bars[B_CHUNK_DONE + s]);

      // ---- chunk c+2 to the prep team (its K, Q tiles were loaded above)
      if (c + 2 < n_chunks && !release_chunk(c + 2)) break;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    // never leave the block with bulk copies still landing in its shared memory
    if (s_issued[0] > 0) mbar_wait_bounded(&bars[B_KQ_FULL + 0], (s_issued[0] - 1) & 1, nullptr, p.status);
    if (s_issued[1] > 0) mbar_wait_bounded(&bars[B_KQ_FULL + 1], (s_issued[1] - 1) & 1, nullptr, p.status);
    if (s_issued[2] > 0) mbar_wait_bounded(&bars[B_V_FULL], (s_issued[2] - 1) & 1, nullptr, p.status);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace tc

// Host launcher: builds the TMA descriptors (3-D views [tokens][H][width] of
// q, k, v with 64 x 1 x 64 boxes, tma_host.h) and launches one CTA per
// (sequence, head, 128-wide dv slice).
bool prefill_tc_supported(const gdn_fwd_params* p) {
  return p->io_dtype == GDN_BF16 && p->dk == tc::DK && p->dv % tc::DVS == 0 &&
         !(p->flags & (GDN_PRECISE | GDN_CHANNEL_GATE));
}

// ------------------------------------------------------------------ segments
// Combine step of the segmented schedule: for one (sequence, head) and
// CMB_COLS columns of dv, S_{p+1} = M_p S_p + B_p for p = 1 .. n_steps,
// starting from S_1 (written by the segment-0 CTAs) and writing every S_p,
// p >= 2, to Sst (slot p-1; M_p and B_p sit in slot p-1 of theirs).  With
// n_steps = n_segs - 2 (output-pass schedule) the last one is S_{n_segs-1};
// with n_steps = n_segs - 1 (corrected schedule) the last one, S_{n_segs}, is
// the final state and goes to S_T (or nowhere when S_T is null).  With Sb
// (corrected schedule) every start state S_1 .. S_{n_segs-1} is also written
// rounded to bf16 into Sb (same layout as Sst), the correction's operand.  The
// products run on the warp-level tensor cores with the 3xTF32 split
// (fp32-level accuracy): warp w owns rows 16w .. 16w+15 of the 128 x CMB_COLS
// block.  M_p (dk x dk) is staged in shared memory by cp.async one step ahead
// (double buffer).
namespace tc {
constexpr int CMB_COLS = 16;                       // columns of dv per CTA
constexpr int CMB_NT = CMB_COLS / 8;               // 8-column mma tiles per warp
constexpr int CMB_MLD = 132;                       // padded row stride of a staged M (floats)
constexpr int CMB_SLD = CMB_COLS + 8;              // padded row stride of the S block (floats)
static_assert(CMB_COLS % 8 == 0 && CMB_SLD % 32 != 0 && (CMB_SLD % 32) % 8 == 0,
              "S-block fragment reads are conflict-free with a row stride of 8 or 24 mod 32");
constexpr uint32_t CMB_SMEM = (2 * DK * CMB_MLD + DK * CMB_SLD) * 4;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(256)
    gdn_segment_combine_kernel(const float* __restrict__ Bws, const float* __restrict__ Mws,
                               float* __restrict__ Sst, float* __restrict__ S_T,
                               __nv_bfloat16* __restrict__ Sb, int H, int dv, int n_segs, int n_part,
                               int n_steps) {
  extern __shared__ __align__(16) float cmb_smem[];
  // launched as a programmatic dependent of the state pass: let the output
  // pass launch, then wait for the state pass before reading its results
  griddep_launch_dependents();
  griddep_wait();
  float* sM0 = cmb_smem;
  float* sM1 = cmb_smem + DK * CMB_MLD;
  float* sS = cmb_smem + 2 * DK * CMB_MLD;         // [128][CMB_SLD], CMB_COLS columns used
  const int ncb = dv / CMB_COLS;
  const int cb = blockIdx.x % ncb;
  const int hh = (blockIdx.x / ncb) % H;
  const int seq = blockIdx.x / (ncb * H);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int g = lane >> 2, q = lane & 3;
  const int r0 = warp * 16;                        // this warp's rows r0 .. r0+15
  const size_t sd = (size_t)DK * dv;               // one state [dk][dv]
  const size_t colb = (size_t)cb * CMB_COLS;
  // slot i holds M_{i+1}, B_{i+1} and S_{i+1}; n_steps products chain S_1 .. S_{n_steps+1}
  // n_part (M, B) slots per sequence
  auto mptr = [&](int pp) { return Mws + (((size_t)seq * n_part + pp) * H + hh) * DK * DK; };
  auto sptr = [&](int pp) -> float* {      // S_{pp+1}
    if (pp <= n_segs - 2) return Sst + (((size_t)seq * (n_segs - 1) + pp) * H + hh) * sd + colb;
    return S_T ? S_T + ((size_t)seq * H + hh) * sd + colb : nullptr;
  };
  auto stage = [&](int pp, float* dst) {
    const float* M = mptr(pp);
#pragma unroll 4
    for (int idx = t; idx < DK * (DK / 4); idx += 256) {
      const int r = idx >> 5, e4 = (idx & 31) * 4;
      cp_async16(dst + r * CMB_MLD + e4, M + (size_t)r * DK + e4);
    }
    cp_async_commit();
  };
  if (n_steps <= 0 && !Sb) return;
  if (n_steps > 0) stage(0, sM0);
  // x[nt][e]: rows r0+g (e = 0, 1) and r0+g+8 (e = 2, 3), columns nt*8 + 2q (+1)
  float x[CMB_NT][4];
#pragma unroll
  for (int nt = 0; nt < CMB_NT; ++nt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const float2 v = *reinterpret_cast<const float2*>(sptr(0) + (size_t)(r0 + g + 8 * hr) * dv + nt * 8 + 2 * q);
      x[nt][2 * hr] = v.x;
      x[nt][2 * hr + 1] = v.y;
    }
  for (int pp = 0;; ++pp) {
    // S_{pp+1} (x) to the operand block, and to Sst (or S_T) unless it came from
    // there; its bf16 copy for the correction (start states only)
    float* dst = (pp > 0) ? sptr(pp) : nullptr;
    __nv_bfloat16* dstb = (Sb && pp <= n_segs - 2)
                              ? Sb + (((size_t)seq * (n_segs - 1) + pp) * H + hh) * sd + colb
                              : nullptr;
#pragma unroll
    for (int nt = 0; nt < CMB_NT; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const float2 v = make_float2(x[nt][2 * hr], x[nt][2 * hr + 1]);
        const int r = r0 + g + 8 * hr, c = nt * 8 + 2 * q;
        if (dst) *reinterpret_cast<float2*>(dst + (size_t)r * dv + c) = v;
        if (dstb) *reinterpret_cast<uint32_t*>(dstb + (size_t)r * dv + c) = pack_bf16x2(v.x, v.y);
        *reinterpret_cast<float2*>(sS + r * CMB_SLD + c) = v;
      }
    if (pp >= n_steps) break;
    const bool prefetch = (pp + 1 < n_steps);
    if (prefetch) stage(pp + 1, ((pp + 1) & 1) ? sM1 : sM0);
    // B is loaded now and added after the product, so its latency is hidden
    const float* B = Bws + (((size_t)seq * n_part + pp) * H + hh) * sd + colb;
    float2 bv[CMB_NT][2];
#pragma unroll
    for (int nt = 0; nt < CMB_NT; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr)
        bv[nt][hr] = *reinterpret_cast<const float2*>(B + (size_t)(r0 + g + 8 * hr) * dv + nt * 8 + 2 * q);
    if (prefetch) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();                                // M_pp and S_pp are in shared memory
    const float* M = (pp & 1) ? sM1 : sM0;
    float acc[CMB_NT][3][4];
#pragma unroll
    for (int nt = 0; nt < CMB_NT; ++nt)
#pragma unroll
      for (int k = 0; k < 3; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][k][e] = 0.f;
#pragma unroll 4
    for (int k0 = 0; k0 < DK; k0 += 8) {
      uint32_t ah[4], al[4];
      split_tf32(M[(r0 + g) * CMB_MLD + k0 + q], ah[0], al[0]);
      split_tf32(M[(r0 + g + 8) * CMB_MLD + k0 + q], ah[1], al[1]);
      split_tf32(M[(r0 + g) * CMB_MLD + k0 + q + 4], ah[2], al[2]);
      split_tf32(M[(r0 + g + 8) * CMB_MLD + k0 + q + 4], ah[3], al[3]);
#pragma unroll
      for (int nt = 0; nt < CMB_NT; ++nt) {
        uint32_t bh[2], bl[2];
        split_tf32(sS[(k0 + q) * CMB_SLD + nt * 8 + g], bh[0], bl[0]);
        split_tf32(sS[(k0 + q + 4) * CMB_SLD + nt * 8 + g], bh[1], bl[1]);
        mma_tf32(acc[nt][0], ah, bh);
        mma_tf32(acc[nt][1], ah, bl);
        mma_tf32(acc[nt][2], al, bh);
      }
    }
#pragma unroll
    for (int nt = 0; nt < CMB_NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[nt][e] = acc[nt][0][e] + (acc[nt][1][e] + acc[nt][2][e]);
      x[nt][0] += bv[nt][0].x;
      x[nt][1] += bv[nt][0].y;
      x[nt][2] += bv[nt][1].x;
      x[nt][3] += bv[nt][1].y;
    }
    __syncthreads();                                // every read of S_pp and M_pp is done
  }
}
// Output correction of the corrected segmented schedule.  Segment p >= 1 of a
// chain ran from a zero state in the state pass and wrote its zero-start
// outputs o^0 into o; its transition slice wrote qhat_i = scale qn_i
// M_{p,i}^T q_i (qn_i = 1/|q_i| with the in-kernel norm, else 1).  The state
// is affine in the start state, so the outputs from the true start state S_p
// are
//     o_i = o^0_i + S_p^T qhat_i,
// which this kernel adds for one (sequence, head, 128-wide dv slice) and a
// tile of up to 128 tokens of one segment.  With the looped block's epilogue
// (output gate, loop residual) the state pass runs without it and this kernel
// applies it to every segment, segment 0 included (whose outputs, run from
// S0, need no correction):
//     o_i <- round(sigmoid(gate_i) round(o_i)) (+ rho (.) h_prev_i, rounded),
// the order in which a gated call followed by loop_residual rounds.
// qhat (K-major A), S_p rounded to bf16 by the combine (MN-major B: rows of
// dk, 64 columns of dv per 128-byte row) and o^0 arrive by TMA in the 128-byte
// swizzle; the product is one tcgen05 MMA chain (M = 128 tokens, N = 128
// columns of dv, K = dk = 128) into tensor memory.  Thread r adds row r of
// the product to o^0 and writes the sum, rounded to bf16, over the o^0 tile;
// the h_prev tile (TMA, into the qhat buffer once the MMA has read it) and the
// gate factors (shared memory) then meet it in coalesced 16-byte rows.  96 KB
// of shared memory: two CTAs per SM.  Launched as a programmatic dependent:
// inputs (gate, rho, and h_prev where no MMA needs the buffer) are read before
// griddepcontrol.wait, anything the state pass or the combine wrote only
// after it.
constexpr int COR_THREADS = 128;
constexpr int COR_ROWS = 128;                      // tokens per tile
constexpr uint32_t COR_TILE = 32768;               // 128 rows x 128 bf16 in two 64-column slabs
constexpr uint32_t COR_OFF_A = 0;                  // qhat, then h_prev
constexpr uint32_t COR_OFF_B = COR_OFF_A + COR_TILE;   // S_p (bf16, MN-major)
constexpr uint32_t COR_OFF_O = COR_OFF_B + COR_TILE;   // o^0, then o^0 + S_p^T qhat
constexpr uint32_t COR_OFF_RHO = COR_OFF_O + COR_TILE; // rho of the slice (128 fp32)
constexpr uint32_t COR_OFF_OG = COR_OFF_RHO + 512;     // gate factor of each row (128 fp32)
constexpr uint32_t COR_OFF_BAR = COR_OFF_OG + 512;     // 4 mbarriers, tmem base, abort flag
constexpr uint32_t COR_SMEM = COR_OFF_BAR + 64 + 1024;

struct CorParams {
  __nv_bfloat16* o;
  const float* gate;             // output-gate logits [tokens][H] (or null)
  const __nv_bfloat16* h_prev;   // loop residual input (or null) and its rho
  const float* rho;
  unsigned* status;
  int H, dv, n_slices, seq_len, seg0_tok, seg_tok, n_segs;
  int tiles_first;               // tiles of segment 0 per (sequence, head, slice): 0 without epilogue
  int tiles_mid, tiles_per_seq;
};

// One 128-token tile of a [tokens][H][width] map (two 64-column slabs, two
// 64-row boxes each).
__device__ __forceinline__ void cor_load_rows(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                              int h, int tok0) {
  tma_load_3d(dst, map, bar, c0, h, tok0);
  tma_load_3d(dst + 8192, map, bar, c0, h, tok0 + 64);
  tma_load_3d(dst + 16384, map, bar, c0 + 64, h, tok0);
  tma_load_3d(dst + 24576, map, bar, c0 + 64, h, tok0 + 64);
}
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(COR_THREADS, 2)
    gdn_segment_correct_kernel(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_sb,
                               const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_h,
                               const CorParams p) {
  extern __shared__ __align__(1024) uint8_t csm_raw[];
  uint8_t* sm = csm_raw;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(sm) & 1023u) {
    if (tid == 0) record_status(p.status, GDN_ERR_CUDA);
    return;
  }
  // [0] qhat and S_p landed, [1] o^0 landed, [2] MMA done, [3] h_prev landed
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + COR_OFF_BAR);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + COR_OFF_BAR + 32);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + COR_OFF_BAR + 36);
  float* s_rho = reinterpret_cast<float*>(sm + COR_OFF_RHO);
  float* s_og = reinterpret_cast<float*>(sm + COR_OFF_OG);
  // block -> (sequence, head, slice, tile); tiles enumerate segment 0 (with the
  // epilogue only), then segments 1 .. n_segs-1
  int bid = (int)blockIdx.x;
  const int tile = bid % p.tiles_per_seq;
  bid /= p.tiles_per_seq;
  const int slice = bid % p.n_slices;
  bid /= p.n_slices;
  const int h = bid % p.H;
  const int seq = bid / p.H;
  const int tps = (p.seg_tok + COR_ROWS - 1) / COR_ROWS;
  int part, i0;
  if (tile < p.tiles_first) {
    part = 0;
    i0 = tile * COR_ROWS;
  } else if (tile - p.tiles_first < p.tiles_mid) {
    part = 1 + (tile - p.tiles_first) / tps;
    i0 = ((tile - p.tiles_first) % tps) * COR_ROWS;
  } else {
    part = p.n_segs - 1;
    i0 = (tile - p.tiles_first - p.tiles_mid) * COR_ROWS;
  }
  const int seg_start = (part == 0) ? 0 : p.seg0_tok + (part - 1) * p.seg_tok;
  const int seg_len = (part == 0) ? p.seg0_tok : min(p.seg_tok, p.seq_len - seg_start);
  const int rows = min(COR_ROWS, seg_len - i0);
  const int tok0 = seq * p.seq_len + seg_start + i0;
  const int col0 = slice * DVS;
  const bool corr = part > 0;                      // start-state share S_p^T qhat
  const bool resid = p.h_prev != nullptr;
  // row of S_p in the [n_seq * (n_segs-1) * H * dk][dv] view of the bf16 start states
  const int sb_row = ((seq * (p.n_segs - 1) + (part - 1)) * p.H + h) * DK;
  const size_t row_elems = (size_t)p.H * p.dv;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(s_tmem, 128);
    tmem_relinquish();
  }
  // inputs first: rho and the gate factors into shared memory
  s_rho[tid] = resid ? __ldg(p.rho + (size_t)h * p.dv + col0 + tid) : 0.f;
  s_og[tid] = (p.gate && tid < rows) ? 1.f / (1.f + __expf(-__ldg(p.gate + (size_t)(tok0 + tid) * p.H + h)))
                                     : 1.f;
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = smem_u32(sm);
  const bool have_rows = rows > 0;
  bool h_issued = false;                           // thread 0: the h_prev copy is in flight
  if (tid == 0 && have_rows) {
    tma_prefetch_desc(&tm_o);
    if (resid) {
      tma_prefetch_desc(&tm_h);
      if (!corr) {                                 // the qhat buffer is free: h_prev now
        mbar_arrive_expect_tx(&bars[3], COR_TILE);
        cor_load_rows(sm + COR_OFF_A, &tm_h, &bars[3], col0, h, tok0);
        h_issued = true;
      }
    }
    if (corr) {
      tma_prefetch_desc(&tm_qh);
      tma_prefetch_desc(&tm_sb);
    }
  }
  griddep_wait();                                  // qhat, o^0 and S_p are written
  if (tid == 0 && have_rows) {
    if (corr) {
      mbar_arrive_expect_tx(&bars[0], 2 * COR_TILE);
      cor_load_rows(sm + COR_OFF_A, &tm_qh, &bars[0], 0, h, tok0);
      tma_load_2d(sm + COR_OFF_B, &tm_sb, &bars[0], col0, sb_row);
      tma_load_2d(sm + COR_OFF_B + 16384, &tm_sb, &bars[0], col0 + 64, sb_row);
    }
    mbar_arrive_expect_tx(&bars[1], COR_TILE);
    cor_load_rows(sm + COR_OFF_O, &tm_o, &bars[1], col0, h, tok0);
  }
  bool ok = have_rows;
  if (ok && corr && warp == 0) {
    const bool okw = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[0], 0, s_abort, p.status));
    tc_fence_after();
    if (okw && elect_one()) {
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        mma_bf16(tmem, kdesc(sbase + COR_OFF_A + (kk >> 2) * 16384 + (kk & 3) * 32),
                 mndesc(sbase + COR_OFF_B + kk * 2048, 16384), idesc_bf16(128, 128, 0, 1), kk > 0);
      mma_commit(&bars[2]);
    }
    __syncwarp();
  }
  if (ok) ok = !__syncthreads_or(!mbar_wait_bounded(&bars[1], 0, s_abort, p.status) || *s_abort != 0);
  if (ok && corr) ok = !__syncthreads_or(!mbar_wait_bounded(&bars[2], 0, s_abort, p.status));
  tc_fence_after();
  if (ok && corr && resid && tid == 0) {
    // the MMA has read qhat: h_prev into its buffer (only the async proxy has
    // touched the buffer, so no proxy fence is needed)
    mbar_arrive_expect_tx(&bars[3], COR_TILE);
    cor_load_rows(sm + COR_OFF_A, &tm_h, &bars[3], col0, h, tok0);
    h_issued = true;
  }
  if (ok && corr) {
    // thread: token row r of the tile; o^0 + S_p^T qhat, rounded to bf16 (the
    // output as it would be stored), replaces o^0 in shared memory
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
    for (int piece = 0; piece < DVS / 32; ++piece) {
      float acc[32];
      tmem_ld32(tmem + lane_off + piece * 32, acc);
      const int cbase = piece * 32;
      const uint32_t slab = (uint32_t)(cbase >> 6) * 16384;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4* ov = reinterpret_cast<uint4*>(sm + COR_OFF_O + slab + sw128_offset(r, (cbase & 63) + c * 8));
        const uint4 x = *ov;
        uint4 v;
        v.x = pack_bf16x2(bf16_lo(x.x) + acc[c * 8 + 0], bf16_hi(x.x) + acc[c * 8 + 1]);
        v.y = pack_bf16x2(bf16_lo(x.y) + acc[c * 8 + 2], bf16_hi(x.y) + acc[c * 8 + 3]);
        v.z = pack_bf16x2(bf16_lo(x.z) + acc[c * 8 + 4], bf16_hi(x.z) + acc[c * 8 + 5]);
        v.w = pack_bf16x2(bf16_lo(x.w) + acc[c * 8 + 6], bf16_hi(x.w) + acc[c * 8 + 7]);
        *ov = v;
      }
    }
  }
  if (ok && resid) ok = !__syncthreads_or(!mbar_wait_bounded(&bars[3], 0, s_abort, p.status));
  if (ok) {
    __syncthreads();
    // coalesced 16-byte rows with the gate and the loop residual; a row past
    // the segment belongs to another segment or sequence and is not touched
    const bool gated = p.gate != nullptr;
#pragma unroll 4
    for (int it = tid; it < COR_ROWS * 16; it += COR_THREADS) {
      const int i = it >> 4, chunk = it & 15;
      if (i < rows) {
        const uint32_t soff = (chunk >> 3) * 16384 + sw128_offset(i, (chunk & 7) * 8);
        uint4 v = *reinterpret_cast<const uint4*>(sm + COR_OFF_O + soff);
        if (gated) {
          const float g = s_og[i];
          v.x = pack_bf16x2(g * bf16_lo(v.x), g * bf16_hi(v.x));
          v.y = pack_bf16x2(g * bf16_lo(v.y), g * bf16_hi(v.y));
          v.z = pack_bf16x2(g * bf16_lo(v.z), g * bf16_hi(v.z));
          v.w = pack_bf16x2(g * bf16_lo(v.w), g * bf16_hi(v.w));
        }
        if (resid) {
          const uint4 y = *reinterpret_cast<const uint4*>(sm + COR_OFF_A + soff);
          const float* rr = s_rho + chunk * 8;
          v.x = pack_bf16x2(fmaf(rr[0], bf16_lo(y.x), bf16_lo(v.x)), fmaf(rr[1], bf16_hi(y.x), bf16_hi(v.x)));
          v.y = pack_bf16x2(fmaf(rr[2], bf16_lo(y.y), bf16_lo(v.y)), fmaf(rr[3], bf16_hi(y.y), bf16_hi(v.y)));
          v.z = pack_bf16x2(fmaf(rr[4], bf16_lo(y.z), bf16_lo(v.z)), fmaf(rr[5], bf16_hi(y.z), bf16_hi(v.z)));
          v.w = pack_bf16x2(fmaf(rr[6], bf16_lo(y.w), bf16_lo(v.w)), fmaf(rr[7], bf16_hi(y.w), bf16_hi(v.w)));
        }
        const size_t off = (size_t)(tok0 + i) * row_elems + (size_t)h * p.dv + col0 + chunk * 8;
        __stcs(reinterpret_cast<uint4*>(p.o + off), v);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && have_rows && !ok) {
    // never leave the block with a bulk copy still landing in its shared memory
    if (corr) mbar_wait_bounded(&bars[0], 0, nullptr, p.status);
    mbar_wait_bounded(&bars[1], 0, nullptr, p.status);
    if (h_issued) mbar_wait_bounded(&bars[3], 0, nullptr, p.status);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Longest-processing-time order of varlen sequences: order[r] is the sequence
// with the r-th largest length (ties by index), so that block r of a one-pass
// launch (blocks are dispatched roughly in index order) takes the longest
// remaining chain.  One CTA sorts (length, index) keys with a bitonic network
// in shared memory; lengths come from cu_seqlens, clamped to [0, 2^31).
constexpr int kLptMaxSeqs = 4096;
constexpr int kLptThreads = 1024;
__global__ void __launch_bounds__(kLptThreads)
    gdn_lpt_order_kernel(const int32_t* __restrict__ cu, int n_seq, int32_t* __restrict__ order) {
  __shared__ unsigned long long key[kLptMaxSeqs];
  int n2 = 1;
  while (n2 < n_seq) n2 <<= 1;
  for (int i = threadIdx.x; i < n2; i += kLptThreads) {
    unsigned long long k = ~0ull;                  // padding sorts last
    if (i < n_seq) {
      long long len = (long long)__ldg(cu + i + 1) - (long long)__ldg(cu + i);
      len = len < 0 ? 0 : (len > 0x7fffffffLL ? 0x7fffffffLL : len);
      k = ((unsigned long long)(0x7fffffffu - (unsigned)len) << 32) | (unsigned)i;
    }
    key[i] = k;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n2; i += kLptThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const unsigned long long a = key[i], b = key[j];
          const bool ascending = (i & size) == 0;
          if ((a > b) == ascending) {
            key[i] = b;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n_seq; i += kLptThreads) order[i] = (int32_t)(key[i] & 0xffffffffu);
}
}  // namespace tc

// Chooses the schedule of a tensor-core prefill: n_segs = 1 is one pass per
// chain; otherwise fixed-length sequences are cut into a segment 0 of seg0_tok
// tokens and n_segs-1 segments of seg_tok.  The cost model counts chunk steps
// on the critical path: waves of CTAs (one CTA per SM) times chunks per CTA.
//   one pass: every chain in one launch.
//   output-pass schedule: the state pass holds segment 0 of every chain (run
//     in full, with outputs) and segments 1 .. n_segs-2 with one transition
//     slice each (no outputs); a combine chains the start states; an output
//     pass recomputes segments 1 .. n_segs-1 from them.
//   corrected schedule: the state pass holds segment 0 and segments
//     1 .. n_segs-1 with their transition slices, all with outputs (the
//     zero-start outputs and the transition's qhat); the combine chains the
//     start states (and the final one); a correction adds S_p^T qhat to the
//     outputs.  Not used when o is h_prev itself: the zero-start outputs are
//     kept in o until the correction, which must still read h_prev.
// A chunk with outputs costs kOutputChunk chunk steps (it adds the output
// products and their epilogue), so segment 0 is made shorter than the others
// in the output-pass schedule.
SegPlan plan_prefill_segments(const gdn_fwd_params* p, int sms) {
  SegPlan plan{1, 0, 0, 0, 0};
  if (!prefill_tc_supported(p) || p->n_seq <= 0 || sms <= 0) return plan;
  if (p->cu_seqlens) {
    // varlen: one pass; with more blocks than one wave, the sequences are
    // launched longest first (an LPT order sorted on the device), so that the
    // longest chains do not start in the last wave
    const long long blocks = (long long)p->n_seq * p->H * (p->dv / tc::DVS);
    plan.lpt = (p->n_seq >= 2 && p->n_seq <= tc::kLptMaxSeqs && blocks > sms) ? 1 : 0;
    return plan;
  }
  if ((p->flags & GDN_SINGLE_PASS) || p->seq_len <= tc::C) return plan;
  constexpr double kOutputChunk = 1.15;   // chunk step of a CTA with outputs / without
  constexpr double kFill = 1.5;           // pipeline fill and drain of a launch wave
  const bool can_correct = !(p->h_prev && p->h_prev == p->o);
  const long long chains = (long long)p->n_seq * p->H;
  const long long slices = p->dv / tc::DVS;
  const int n_chunks = (p->seq_len + tc::C - 1) / tc::C;
  auto waves = [&](long long ctas) { return (double)((ctas + sms - 1) / sms); };
  const double one_pass = waves(chains * slices) * (n_chunks * kOutputChunk + kFill);
  double best = 0.0;
  SegPlan cand{1, 0, 0, 0, 0};
  auto consider = [&](double cost, const SegPlan& c) {
    if (cand.n_segs == 1 || cost < best) {
      best = cost;
      cand = c;
    }
  };
  for (int seg = 1; seg < n_chunks; ++seg) {
    for (int seg0 = seg; seg0 >= 1 && seg0 >= seg - 4; --seg0) {
      if (seg0 >= n_chunks) continue;
      const int P = 1 + (n_chunks - seg0 + seg - 1) / seg;
      // output-pass schedule; a combine step costs about 0.8 of a chunk step
      const double cost =
          waves(chains * (slices + (long long)(P - 2) * (slices + 1))) *
              (fmax(seg0 * kOutputChunk, (double)seg) + kFill) +
          waves(chains * (P - 1) * slices) * (seg * kOutputChunk + kFill) + (P > 2 ? 0.8 * (P - 2) + 0.5 : 0.0);
      consider(cost, SegPlan{P, seg * tc::C, seg0 * tc::C, 0, 0});
      if (can_correct && seg0 == seg) {
        // corrected schedule: every state-pass CTA has outputs; the correction
        // costs about 1.5 chunk steps
        const double cc = waves(chains * (slices + (long long)(P - 1) * (slices + 1))) *
                              (seg * kOutputChunk + kFill) + 0.8 * (P - 1) + 0.5 + 1.5;
        consider(cc, SegPlan{P, seg * tc::C, seg0 * tc::C, 0, 1});
      }
    }
  }
  // segmented only when clearly cheaper than one pass
  return (cand.n_segs > 1 && best < 0.85 * one_pass) ? cand : plan;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of a segmented schedule: [B | M | S | qhat | Sb] with B and M for
// n_part segments (n_segs-2 in the output-pass schedule, n_segs-1 in the
// corrected one), start states S_1 .. S_{n_segs-1}, and for the corrected
// schedule qhat [total_tokens][H][dk] bf16 and the start states in bf16;
// each buffer 256-byte aligned.
size_t prefill_segment_workspace(const gdn_fwd_params* p, const SegPlan& plan) {
  if (plan.lpt) return align256((size_t)p->n_seq * sizeof(int32_t));
  if (plan.n_segs <= 1) return 0;
  const size_t sd = (size_t)p->H * tc::DK * p->dv * sizeof(float);
  const size_t md = (size_t)p->H * tc::DK * tc::DK * sizeof(float);
  const size_t n = (size_t)p->n_seq;
  const size_t n_part = plan.corrected ? plan.n_segs - 1 : plan.n_segs - 2;
  const size_t qh = plan.corrected ? (size_t)p->total_tokens * p->H * tc::DK * 2 : 0;
  const size_t sb = plan.corrected ? n * (plan.n_segs - 1) * sd / 2 : 0;
  return align256(n * n_part * sd) + align256(n * n_part * md) + align256(n * (plan.n_segs - 1) * sd) +
         align256(qh) + align256(sb);
}

// Launch configuration; `dependent` launches with programmatic stream
// serialization (the grid may start while the previous one in the stream is
// finishing and orders its reads of that grid's results by griddep_wait()).
struct LaunchCfg {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  LaunchCfg(unsigned blocks, unsigned threads, size_t smem, cudaStream_t stream, bool dependent) {
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
  }
};

static gdn_status tc_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const tc::Params& kp, long long blocks, cudaStream_t stream,
                            bool dependent = false) {
  if (blocks <= 0) return GDN_OK;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  LaunchCfg lc((unsigned)blocks, tc::THREADS, tc::SMEM_BYTES, stream, dependent);
  const bool epi = kp.gate != nullptr || kp.h_prev != nullptr;
  const cudaError_t e = epi ? cudaLaunchKernelEx(&lc.cfg, tc::gdn_prefill_tc_kernel<true>, mq, mk, mv, kp)
                            : cudaLaunchKernelEx(&lc.cfg, tc::gdn_prefill_tc_kernel<false>, mq, mk, mv, kp);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status launch_prefill_tc(const gdn_fwd_params* p, unsigned* status, const SegPlan& plan, void* ws,
                             cudaStream_t stream) {
  static std::atomic<bool> attr_set[kMaxDevices], attr_set_epi[kMaxDevices];
  if (smem_attr_once(attr_set, tc::gdn_prefill_tc_kernel<false>, tc::SMEM_BYTES) != cudaSuccess ||
      smem_attr_once(attr_set_epi, tc::gdn_prefill_tc_kernel<true>, tc::SMEM_BYTES) != cudaSuccess)
    return GDN_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, p->q, p->dk, p->H, p->total_tokens) ||
      !make_map(&mk, p->k, p->dk, p->H, p->total_tokens) ||
      !make_map(&mv, p->v, p->dv, p->H, p->total_tokens))
    return GDN_ERR_CUDA;
  tc::Params kp;
  kp.a = p->a;
  kp.b = p->b;
  kp.S0 = p->S0;
  kp.S_T = p->S_T;
  kp.o = static_cast<__nv_bfloat16*>(p->o);
  kp.cu_seqlens = p->cu_seqlens;
  kp.status = status;
  kp.gate = p->gate;
  kp.h_prev = static_cast<const __nv_bfloat16*>(p->h_prev);
  kp.rho = p->rho;
  kp.n_seq = p->n_seq;
  kp.seq_len = p->seq_len;
  kp.total_tokens = p->total_tokens;
  kp.H = p->H;
  kp.dv = p->dv;
  kp.n_slices = p->dv / tc::DVS;
  kp.scale = p->scale;
  kp.flags = p->flags;
  kp.mode = 0;
  kp.n_segs = 1;
  kp.seg_tok = 0;
  kp.seg0_tok = 0;
  kp.Bws = kp.Mws = nullptr;
  kp.Sst = nullptr;
  kp.qhat = nullptr;
  kp.order = nullptr;
  const long long chains = (long long)p->n_seq * p->H;
  if (plan.lpt) {
    int32_t* order = static_cast<int32_t*>(ws);
    tc::gdn_lpt_order_kernel<<<1, tc::kLptThreads, 0, stream>>>(p->cu_seqlens, p->n_seq, order);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    kp.order = order;
  }
  if (plan.n_segs <= 1) return tc_launch(mq, mk, mv, kp, chains * kp.n_slices, stream);

  // segmented: workspace = [B | M | S_1 .. S_{P-1} | qhat] (prefill_segment_workspace)
  const int P = plan.n_segs;
  const int n_part = plan.corrected ? P - 1 : P - 2;
  const size_t sd = (size_t)p->H * tc::DK * p->dv * sizeof(float);
  const size_t md = (size_t)p->H * tc::DK * tc::DK * sizeof(float);
  char* w = static_cast<char*>(ws);
  kp.Bws = reinterpret_cast<float*>(w);
  w += align256((size_t)p->n_seq * n_part * sd);
  kp.Mws = reinterpret_cast<float*>(w);
  w += align256((size_t)p->n_seq * n_part * md);
  kp.Sst = reinterpret_cast<float*>(w);
  w += align256((size_t)p->n_seq * (P - 1) * sd);
  kp.qhat = plan.corrected ? reinterpret_cast<__nv_bfloat16*>(w) : nullptr;
  w += plan.corrected ? align256((size_t)p->total_tokens * p->H * tc::DK * 2) : 0;
  __nv_bfloat16* Sb = plan.corrected ? reinterpret_cast<__nv_bfloat16*>(w) : nullptr;
  kp.n_segs = P;
  kp.seg_tok = plan.seg_tok;
  kp.seg0_tok = plan.seg0_tok;
  kp.mode = plan.corrected ? 3 : 1;
  // corrected schedule: the output gate and the loop residual are applied by
  // the correction kernel (to every segment), not in the state pass's chunk loop
  const bool epilogue = kp.gate != nullptr || kp.h_prev != nullptr;
  if (plan.corrected) {
    kp.gate = nullptr;
    kp.h_prev = nullptr;
    kp.rho = nullptr;
  }
  gdn_status st =
      tc_launch(mq, mk, mv, kp, chains * (kp.n_slices + (long long)n_part * (kp.n_slices + 1)), stream);
  if (st != GDN_OK) return st;
  // combine: start states S_2 .. S_{P-1} (and S_T in the corrected schedule,
  // with every start state also in bf16 for the correction)
  const int n_steps = plan.corrected ? (p->S_T ? P - 1 : P - 2) : P - 2;
  if (n_steps > 0 || plan.corrected) {
    const long long cblocks = chains * (p->dv / tc::CMB_COLS);
    if (cblocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    static std::atomic<bool> cmb_attr_set[kMaxDevices];
    if (smem_attr_once(cmb_attr_set, tc::gdn_segment_combine_kernel, tc::CMB_SMEM) != cudaSuccess)
      return GDN_ERR_CUDA;
    LaunchCfg lc((unsigned)cblocks, 256, tc::CMB_SMEM, stream, /*dependent=*/true);
    if (cudaLaunchKernelEx(&lc.cfg, tc::gdn_segment_combine_kernel, (const float*)kp.Bws,
                           (const float*)kp.Mws, kp.Sst, plan.corrected ? p->S_T : nullptr, Sb, p->H,
                           p->dv, P, n_part, n_steps) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  if (!plan.corrected) {
    kp.mode = 2;
    return tc_launch(mq, mk, mv, kp, chains * (P - 1) * kp.n_slices, stream, /*dependent=*/true);
  }
  // correction of the outputs of segments 1 .. P-1, and the epilogue of all
  CUtensorMap mqh, msb, mo, mh;
  if (!make_map(&mqh, kp.qhat, tc::DK, p->H, p->total_tokens) ||
      !make_map_2d(&msb, Sb, p->dv, (long long)p->n_seq * (P - 1) * p->H * tc::DK, 64, 128) ||
      !make_map(&mo, p->o, p->dv, p->H, p->total_tokens) ||
      !make_map(&mh, p->h_prev ? p->h_prev : p->o, p->dv, p->H, p->total_tokens))
    return GDN_ERR_CUDA;
  tc::CorParams cp;
  cp.o = kp.o;
  cp.gate = p->gate;
  cp.h_prev = static_cast<const __nv_bfloat16*>(p->h_prev);
  cp.rho = p->rho;
  cp.status = status;
  cp.H = p->H;
  cp.dv = p->dv;
  cp.n_slices = kp.n_slices;
  cp.seq_len = p->seq_len;
  cp.seg0_tok = plan.seg0_tok;
  cp.seg_tok = plan.seg_tok;
  cp.n_segs = P;
  const int tps = (plan.seg_tok + tc::COR_ROWS - 1) / tc::COR_ROWS;
  const int last_len = p->seq_len - plan.seg0_tok - (P - 2) * plan.seg_tok;
  cp.tiles_first = epilogue ? (plan.seg0_tok + tc::COR_ROWS - 1) / tc::COR_ROWS : 0;
  cp.tiles_mid = (P - 2) * tps;
  cp.tiles_per_seq = cp.tiles_first + cp.tiles_mid + (last_len + tc::COR_ROWS - 1) / tc::COR_ROWS;
  const long long cor_blocks = chains * kp.n_slices * cp.tiles_per_seq;
  if (cor_blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  static std::atomic<bool> cor_attr_set[kMaxDevices];
  if (smem_attr_once(cor_attr_set, tc::gdn_segment_correct_kernel, tc::COR_SMEM) != cudaSuccess)
    return GDN_ERR_CUDA;
  LaunchCfg lc((unsigned)cor_blocks, tc::COR_THREADS, tc::COR_SMEM, stream, /*dependent=*/true);
  return cudaLaunchKernelEx(&lc.cfg, tc::gdn_segment_correct_kernel, mqh, msb, mo, mh, cp) == cudaSuccess
             ? GDN_OK
             : GDN_ERR_CUDA;
}

}  // namespace gdn
