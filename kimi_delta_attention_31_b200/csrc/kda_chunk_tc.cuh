// kda_chunk_tc.cuh -- tensor-core (tcgen05 / TMEM) chunkwise KDA prefill for
// bf16 q, k, v with dk = dv = 128 and C = 64 tokens per chunk.
//
// The schedule ("Deriving Kimi Delta Attention from scratch", section 6,
// chunked mode; "Linear / sparse attention" tutorial, section 5.3 WY
// representation and section 6.2 chunk skeleton).  Within a chunk entering
// with state S, with chunk-relative cumulative log-decays G (fp32):
//   A_rj = beta_r sum_c k_rc k_jc e^{G_rc - G_jc}  (j < r),
//   P_rj =        sum_c q_rc k_jc e^{G_rc - G_jc}  (j <= r),
//   T = (I + A)^{-1},  W = T diag(beta) (K o e^G),  U = T diag(beta) V,
//   E = U - W S,  O = (Q o e^G) S + P E,
//   S <- Diag(e^{G_last}) S + (K o e^{G_last - G})^T E.
// Everything left of "S" is chunk-local and parallel over chunks; only the
// last three lines carry the state.  Two kernels:
//
//  1. kda_tc_chunk_local_kernel -- one CTA per (chunk, head), all chunks in
//     parallel.  Builds the decay-scaled bf16 operands in shared memory,
//     computes [A; P] with one tcgen05 MMA (M=128, N=160, K=128) into TMEM,
//     inverts I + A in fp32 (blocked by 16), forms W^T and U^T (two MMAs),
//     and writes a 74,240-byte per-chunk image already laid out as the
//     state pass's MMA operands.
//  2. kda_tc_state_pass_kernel -- persistent, one CTA per SM, one (sequence,
//     head) unit at a time, chunks in order.  The fp32 state lives in
//     registers (thread = state row x 64 columns); per chunk one bulk copy
//     brings the image in (double-buffered) and two MMA groups run:
//       X = [-I; 0] U + [W; Q e^G] S_bf16  -> rows 0..63 = -E, rows 64..127 = Q e^G S
//       Y = Kbar^T E,  X += [*; P] E       -> S <- gamma o S + Y,  O = rows 64..127 of X.
//
// Overflow-free decay factors: A and P are never formed from e^{G} and
// e^{-G} over the whole chunk.  The chunk is split into four 16-token blocks;
// with a_r = e^{G_r - G_start(block)} and b_r = e^{G_end(block) - G_r} (both
// in (0, 1]), an off-diagonal block pair (I > J) uses
//   left  = k_r a_r            (row block I, reference = start of block I)
//   right = k_j b_j e^{G_start(I) - G_end(J)}   (<= 1)
// and a diagonal block uses left = k_r a_r, right = k_j b_j e^{G_start - G_end}
// (= k_j / a_j).  The only factor above 1 is e^{-(block log-decay)}, finite as
// long as every channel's log-decay over one 16-token block is >= -80.
#pragma once
#include <algorithm>
#include "kda_common.cuh"
#include "tc_ptx.cuh"

namespace kda {

constexpr bool kTcPathBuilt = true;
constexpr int kTcLaunches = 2;

namespace tc {

using bf16 = __nv_bfloat16;
constexpr int C = 64;   // tokens per chunk
constexpr int D = 128;  // dk = dv

// -softplus(a) = -(max(a, 0) + log(1 + y)), y = e^{-|a|} in (0, 1], on the
// SFU's exp2 and log2 instead of log1pf, for the bf16 tensor-core kernels'
// gate logits: log(1 + y) directly when y >= 2^-8 (1 + y then rounds by at
// most 2^-24 of itself), else the series y - y^2/2 + y^3/3, whose error is
// below y^4/4 < 2^-34.  Its largest absolute error over a in [-40, 40] is
// about 5e-7, so a chunk's gate sum (at most 64 terms) is off by a few 1e-6
// at most, far inside those kernels' tolerance.  The fp32 path and the
// backward keep log1pf.
__device__ __forceinline__ float neg_softplus_sfu(float a) {
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  const float y = ptx::ex2(-fabsf(a) * kLog2e);
  const float l = y >= 0.00390625f ? __log2f(1.f + y) * kLn2 : y * (1.f - y * (0.5f - y * (1.f / 3.f)));
  return -(fmaxf(a, 0.f) + l);
}

// Per (chunk, head) image: written by the chunk-local kernel, copied in one
// piece by the state pass.  Offsets in bytes; every piece 1024-aligned.
constexpr uint32_t IMG_P = 0;       // P     K-major [64 r][64 j]                 8192
constexpr uint32_t IMG_U = 8192;    // U^T   K-major [128 dv][64 j]               16384
constexpr uint32_t IMG_A1 = 24576;  // [W;Q e^G] MN-major: 2 panels [128 dk][64 tok] 32768
constexpr uint32_t IMG_KB = 57344;  // Kbar  MN-major: 2 panels [64 tok][64 dk]   16384
constexpr uint32_t IMG_G = 73728;   // gamma = e^{G_last}, fp32 [128]             512
constexpr uint32_t IMG_BYTES = 74240;

// chunk-local kernel shared memory (dynamic, 1024-aligned base)
// L3 is two K-panels of 128 rows: rows 0..63 (the K part) of each panel are
// bytes [0, 8K) and [16K, 24K); the Q part fills [8K, 16K) and [24K, 32K).
constexpr uint32_t KA_L3 = 0;       // [K a; Q a]  K-major [128][128] (2 K-panels)  32768
constexpr uint32_t KA_RB = 32768;   // right operands K-major [160][128]          40960
constexpr uint32_t KA_TT = 8192;    // after the first MMA: T diag(beta) bf16 (Q part of panel 0) 8192
constexpr uint32_t KA_PT = 24576;   //                      P bf16 K-major (Q part of panel 1)  8192
// P, U^T and W^T are staged at KA_PT .. KA_PT + 40960 (U^T and W^T over A and T,
// after the second MMA) in image order and leave in one bulk store.
constexpr uint32_t KA_IMG_STAGE = KA_PT;
constexpr uint32_t KA_AS = 32768;   //                      A fp32 [64][68], then T (over RB)  17408
constexpr uint32_t KA_XK = 73728;   // K o e^G  MN-major 2 panels [64][64] (block path) 16384
constexpr uint32_t KA_BV = 90112;   // V        MN-major 2 panels [64][64]       16384
constexpr uint32_t KA_BYTES = 106496;
constexpr uint32_t KA_DYN = KA_BYTES + 1024;

// state-pass kernel shared memory (two CTAs per SM).  The image arrives in
// three parts, each reloaded as soon as its last reader is done: [W; Q e^G]
// (read by the first MMA), U^T (read by the first epilogue, then overwritten
// by E), and P + Kbar + gamma (read by the second MMA group).  P sits right
// after the state operand, whose last 8 KB serve as the unused upper half of
// the [*; P] operand.
constexpr uint32_t KB_SB = 0;        // S bf16 MN-major 2 panels [128 dk][64 dv]          32768
constexpr uint32_t KB_P = 32768;     // P K-major [64 r][64 j]                             8192
constexpr uint32_t KB_UE = 40960;    // U^T K-major [128 dv][64 j], then E MN-major 2 x [64 j][64 dv] 16384
constexpr uint32_t KB_WQ = 57344;    // [W; Q e^G] MN-major 2 panels [128 dk][64 tok]      32768
constexpr uint32_t KB_KG = 90112;    // Kbar MN-major 2 panels [64 tok][64 dk], gamma fp32 [128] 16896
constexpr uint32_t KB_BYTES = KB_KG + 16896;
constexpr uint32_t KB_DYN = KB_BYTES + 1024;

// 1024-byte aligned start inside the dynamic shared buffer.  Offsetting the
// array (not casting through an integer) keeps the pointer in the shared
// address space, so the compiler emits st.shared/ld.shared and can reorder
// global loads around them.
#define KDA_ALIGNED_DSMEM(name, raw) \
  uint8_t* name = (raw) + ((1024u - (ptx::smem_u32(raw) & 1023u)) & 1023u)
__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 r;
  r.x = ptx::pack_bf16x2(x[0], x[1]);
  r.y = ptx::pack_bf16x2(x[2], x[3]);
  r.z = ptx::pack_bf16x2(x[4], x[5]);
  r.w = ptx::pack_bf16x2(x[6], x[7]);
  return r;
}

// Packed layout: chunk `ci` (chunks numbered over all sequences in order,
// C tokens each, restarting at every sequence) -> token start and length.
// Executed by one full warp; returns false when ci is past the last chunk.
__device__ bool locate_chunk_warp(const int32_t* cu, int num_seqs, long long ci, long long* s_out,
                                  int* cn_out) {
  const int lane = threadIdx.x & 31;
  long long acc = 0;
  for (int base = 0; base < num_seqs; base += 32) {
    const int m = base + lane;
    long long st = 0, en = 0, nch = 0;
    if (m < num_seqs) {
      st = cu[m];
      en = cu[m + 1];
      nch = (en - st + C - 1) / C;
    }
    long long incl = nch;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    const long long excl = incl - nch;
    const bool mine = m < num_seqs && ci >= acc + excl && ci < acc + incl;
    const unsigned ball = __ballot_sync(0xffffffffu, mine);
    if (ball) {
      const int src = __ffs(ball) - 1;
      const long long s = __shfl_sync(0xffffffffu, st + (ci - acc - excl) * C, src);
      const long long e = __shfl_sync(0xffffffffu, en, src);
      *s_out = s;
      *cn_out = (int)min((long long)C, e - s);
      return true;
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  return false;
}

// Number of chunks of sequences 0..n-1 (one full warp; same result on all lanes).
__device__ long long chunks_before_warp(const int32_t* cu, int n) {
  const int lane = threadIdx.x & 31;
  long long acc = 0;
  for (int base = 0; base < n; base += 32) {
    const int m = base + lane;
    long long x = m < n ? (long long)(cu[m + 1] - cu[m] + C - 1) / C : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    acc += x;
  }
  return acc;
}


// ---------------------------------------------------------------------------
// Kernel 1: chunk-local work, one CTA (256 threads) per (chunk, head).
// Operand building: thread t owns channels 8 (t mod 16) .. + 7 of rows
// 4 (t / 16) .. + 3, so every global load and shared store moves 16 bytes.
// ---------------------------------------------------------------------------
// A chunk whose every channel keeps its log-decay over the whole chunk above
// this bound takes the single-reference form (left K o e^{G}, right K o e^{-G}):
// both factors and every product stay inside the fp32 / bf16 exponent range.
constexpr float kChunkRefMinG = -80.f;
constexpr int AS_LD = 68;          // row stride (floats) of A and T in fp32

// acc (16 x 16 as two m16n8 halves) += X (16 x 16, fp32, row stride ldx) * Y (16 x 16,
// row stride ldy), one warp, TF32 operands with fp32 accumulation.
__device__ __forceinline__ void warp_gemm16(float (&acc)[2][4], const float* xp, int ldx, const float* yp,
                                            int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int kh = 0; kh < 2; ++kh) {
    const uint32_t a[4] = {ptx::to_tf32(xp[g * ldx + 8 * kh + t]), ptx::to_tf32(xp[(g + 8) * ldx + 8 * kh + t]),
                           ptx::to_tf32(xp[g * ldx + 8 * kh + t + 4]),
                           ptx::to_tf32(xp[(g + 8) * ldx + 8 * kh + t + 4])};
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      const uint32_t b[2] = {ptx::to_tf32(yp[(8 * kh + t) * ldy + 8 * nh + g]),
                             ptx::to_tf32(yp[(8 * kh + t + 4) * ldy + 8 * nh + g])};
      ptx::mma_tf32_m16n8k8(acc[nh], a, b);
    }
  }
}
// The same product with each operand split as tf32 hi + lo (x = hi + lo to
// about 2^-22): acc += Xlo Yhi + Xhi Ylo + Xhi Yhi, three TF32 MMAs per step,
// about fp32 accuracy.  For blocks of A whose entries are large (near-parallel
// keys), where the block products cancel and TF32 rounding would not average
// out.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = ptx::to_tf32(x);
  lo = ptx::to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void warp_gemm16_3x(float (&acc)[2][4], const float* xp, int ldx, const float* yp,
                                               int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int kh = 0; kh < 2; ++kh) {
    uint32_t ah[4], al[4];
    split_tf32(xp[g * ldx + 8 * kh + t], ah[0], al[0]);
    split_tf32(xp[(g + 8) * ldx + 8 * kh + t], ah[1], al[1]);
    split_tf32(xp[g * ldx + 8 * kh + t + 4], ah[2], al[2]);
    split_tf32(xp[(g + 8) * ldx + 8 * kh + t + 4], ah[3], al[3]);
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      uint32_t bh[2], bl[2];
      split_tf32(yp[(8 * kh + t) * ldy + 8 * nh + g], bh[0], bl[0]);
      split_tf32(yp[(8 * kh + t + 4) * ldy + 8 * nh + g], bh[1], bl[1]);
      ptx::mma_tf32_m16n8k8(acc[nh], al, bh);
      ptx::mma_tf32_m16n8k8(acc[nh], ah, bl);
      ptx::mma_tf32_m16n8k8(acc[nh], ah, bh);
    }
  }
}
// An entry of A at least this large switches the chunk's block products to
// warp_gemm16_3x (keys this close to parallel do not occur by chance in 128
// dimensions; repeated or near-duplicate keys do).
constexpr float kSolveAccurateA = 0.5f;

__device__ __forceinline__ void warp_store16(float* dp, int ldd, const float (&acc)[2][4], float scale, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    dp[g * ldd + 8 * nh + 2 * t] = scale * acc[nh][0];
    dp[g * ldd + 8 * nh + 2 * t + 1] = scale * acc[nh][1];
    dp[(g + 8) * ldd + 8 * nh + 2 * t] = scale * acc[nh][2];
    dp[(g + 8) * ldd + 8 * nh + 2 * t + 1] = scale * acc[nh][3];
  }
}

__device__ __forceinline__ void unpack8(uint4 w, float* x) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void normalise_rows(float* kv, float* qv, float nk, float nq) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    kv[e] *= nk;
    qv[e] *= nq;
  }
}

// Phase 4 on the single-reference path: TMEM columns [tm, tm + 64) hold, in
// lanes 0..63, A'_rj and in lanes 64..127, P'_rj (the other way round when
// `p_first`).  Writes A = beta_r A'_rj (j < r, fp32, row stride AS_LD) and P
// (j <= r, bf16 K-major 128-byte swizzled, zero above the diagonal).  Returns
// whether some |A_rj| this thread wrote is at least kSolveAccurateA.  Eight
// warps; `warp` is the warp's index in the CTA (its TMEM lane quarter is
// warp mod 4) and `w8` its index in the group of eight (which 32 columns it takes).
__device__ __forceinline__ bool scatter_single_ref(uint32_t tm, const float* s_beta, float* As, uint8_t* Pt,
                                                   int warp, int w8, int lane, bool p_first = false) {
  const int qd = warp & 3, ch = w8 >> 2;
  const int rho = 32 * qd + lane, r = rho & 63, j0 = 32 * ch;
  float x[32];
  const uint32_t ta = tm + ((uint32_t)(32 * qd) << 16) + j0;
  ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
  ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
  ptx::tmem_wait_ld();
  if ((rho < 64) != p_first) {  // warp-uniform
    const float br = s_beta[r];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = (j0 + e < r) ? br * x[e] : 0.f;
    float4* dst = reinterpret_cast<float4*>(As + r * AS_LD + j0);
    float mx = 0.f;
#pragma unroll
    for (int v4 = 0; v4 < 8; ++v4) {
      dst[v4] = make_float4(x[4 * v4], x[4 * v4 + 1], x[4 * v4 + 2], x[4 * v4 + 3]);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x[4 * v4]), fabsf(x[4 * v4 + 1])), fmaxf(fabsf(x[4 * v4 + 2]), fabsf(x[4 * v4 + 3]))));
    }
    return mx >= kSolveAccurateA;
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = (j0 + e <= r) ? x[e] : 0.f;
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) *reinterpret_cast<uint4*>(Pt + ptx::sw128_chunk(r, 4 * ch + k8)) = pack8(x + 8 * k8);
    return false;
  }
}

// acc <- the 16 x 16 fp32 block at dp (row stride ldd), in the C-fragment
// layout of warp_gemm16.
__device__ __forceinline__ void warp_load16(float (&acc)[2][4], const float* dp, int ldd, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    const float2 a = *reinterpret_cast<const float2*>(dp + g * ldd + 8 * nh + 2 * t);
    const float2 b = *reinterpret_cast<const float2*>(dp + (g + 8) * ldd + 8 * nh + 2 * t);
    acc[nh][0] = a.x;
    acc[nh][1] = a.y;
    acc[nh][2] = b.x;
    acc[nh][3] = b.y;
  }
}
// Block (I, J) of T diag(beta), T_IJ = scale * acc (C-fragment layout): bf16
// hi into Tt (K-major [64 r][64 j], 128-byte swizzle), and lo = bf16(x - hi)
// returned in lo[] (the words t_beta_store_lo writes) when the caller keeps a
// lo part.
__device__ __forceinline__ void t_beta_hi(const float (&acc)[2][4], float scale, const float* s_beta, int I, int J,
                                          uint8_t* Tt, uint32_t (&lo)[4], int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    const float2 b = *reinterpret_cast<const float2*>(s_beta + 16 * J + 8 * nh + 2 * t);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = 16 * I + g + 8 * hh;
      const float x0 = scale * acc[nh][2 * hh] * b.x, x1 = scale * acc[nh][2 * hh + 1] * b.y;
      const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
      const float2 hf = __bfloat1622float2(h);
      *reinterpret_cast<__nv_bfloat162*>(Tt + r * 128 + ((((2 * J + nh) ^ r) & 7) << 4) + 4 * t) = h;
      lo[2 * nh + hh] = ptx::pack_bf16x2(x0 - hf.x, x1 - hf.y);
    }
  }
}
__device__ __forceinline__ void t_beta_store_lo(const uint32_t (&lo)[4], int I, int J, uint8_t* Tlo, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = 16 * I + g + 8 * hh;
      *reinterpret_cast<uint32_t*>(Tlo + r * 128 + ((((2 * J + nh) ^ r) & 7) << 4) + 4 * t) = lo[2 * nh + hh];
    }
}
// Zeroes the 16 x 16 bf16 block (I, J) of a K-major [64][64] swizzled tile (one warp).
__device__ __forceinline__ void zero_block16(uint8_t* Tx, int I, int J, int lane) {
  *reinterpret_cast<uint4*>(Tx + ptx::sw128_chunk(16 * I + (lane >> 1), 2 * J + (lane & 1))) =
      make_uint4(0u, 0u, 0u, 0u);
}

// Phase 5: T = (I + A)^{-1} (A strictly lower, fp32 in As, row stride AS_LD),
// blocked by 16, computed in place over A, and T diag(beta) in bf16 (K-major
// [64 r][64 j], 128-byte swizzle) into Tt.  The diagonal blocks by forward
// substitution in fp32, one thread per column of T holding the column's 16
// rows in registers (rows of A are broadcast loads).  The off-diagonal blocks
// by levels over eight warps: with the 32 x 32 halves TA = T[0:32, 0:32] and
// TB = T[32:64, 32:64] (the inverse of a block lower-triangular matrix),
//   level 1   T10 = -T11 A10 T00,  T32 = -T33 A32 T22,  and A20 T00, A30 T00,
//             A21 T11, A31 T11
//   level 2   X = A[32:64, 0:32] TA (its other two blocks), T21 = -T22 X21,
//             T31 = -(T32 X21 + T33 X31)
//   level 3   T20 = -T22 X20,  T30 = -(T32 X20 + T33 X30)
// so that no chain is longer than two 16 x 16 products per level.  Only the
// diagonal blocks, T10 and T32 are read again: they overwrite their blocks of
// A once no other warp reads those; the intermediate blocks live in the upper
// blocks of As.  The products are TF32 warp MMAs with fp32 accumulation, in
// split TF32 (about fp32 accuracy) when `accurate` (some |A_rj| >=
// kSolveAccurateA, voted by the caller).  Each block of T diag(beta) goes to
// bf16 as soon as it is final.  kPrecise (for chunks where some |A_rj| >=
// kSolveAccurateA, see solve_t_beta_precise) adds two things: split-TF32
// products (about fp32 accuracy), and T diag(beta) split as hi + lo,
// hi = bf16(x) into Tt and lo = bf16(x - hi) into Tlo (its own buffer, same
// layout), so that a pair of bf16 MMAs uses it to about 2^-16.  Without it the
// products are plain TF32 and only hi is written (Tlo is not touched).
// 256 threads: t in [0, 256), w = t / 32; `sync` is their barrier.  Tt and
// Tlo are first written after the first barrier; the caller's barrier after
// the call makes everything visible.  Warp 7 calls `idle()` (all its lanes)
// after its level-1 work: it has nothing more to do in the call.
template <bool kPrecise, typename Sync, typename Idle>
__device__ __forceinline__ void solve_t_beta(float* As, const float* s_beta, uint8_t* Tt, uint8_t* Tlo, int t,
                                             int w, int lane, Sync sync, Idle idle) {
  if (t < 64) {  // diagonal blocks: forward substitution, one thread per column
    const int jj = t & 15, o = t & 48;
    float x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = (m == jj) ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      const float* arow = As + (o + i) * AS_LD + o;
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if (4 * q4 < i) {
          const float4 a4 = *reinterpret_cast<const float4*>(arow + 4 * q4);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int m = 4 * q4 + e;
            if (m < i) {
              if (m & 1) acc1 = fmaf(av[e], x[m], acc1);
              else acc0 = fmaf(av[e], x[m], acc0);
            }
          }
        }
      }
      if (i > jj) x[i] = -(acc0 + acc1);
    }
    __syncwarp();  // the block's 16 threads (one half-warp) have read its rows of A
#pragma unroll
    for (int i = 0; i < 16; ++i) As[(o + i) * AS_LD + o + jj] = x[i];
  }
  sync();  // diagonal blocks of T visible
  auto gemm = [&](float (&acc)[2][4], const float* xp, const float* yp) {  // acc += X Y
    if (kPrecise) warp_gemm16_3x(acc, xp, AS_LD, yp, AS_LD, lane);
    else warp_gemm16(acc, xp, AS_LD, yp, AS_LD, lane);
  };
  auto blk = [As](int I, int J) { return As + 16 * I * AS_LD + 16 * J; };
  auto clear = [](float (&acc)[2][4]) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[i][k] = 0.f;
  };
  auto final_block = [&](const float (&acc)[2][4], float scale, int I, int J) {
    uint32_t lo[4];
    t_beta_hi(acc, scale, s_beta, I, J, Tt, lo, lane);
    if (kPrecise) t_beta_store_lo(lo, I, J, Tlo, lane);
  };
  // intermediate blocks, in the upper blocks of As
  float* m10 = blk(0, 1);  // A10 T00
  float* m32 = blk(2, 3);  // A32 T22
  float* x20 = blk(0, 2);  // A20 T00, then X20 = A20 T00 + A21 T10
  float* x30 = blk(0, 3);  // A30 T00, then X30 = A30 T00 + A31 T10
  float* x21 = blk(1, 2);  // X21 = A21 T11
  float* x31 = blk(1, 3);  // X31 = A31 T11
  float acc[2][4];
  // ---- level 1
  if (w < 2) {  // T10 (w = 0), T32 (w = 1), each over its block of A
    const int I = 2 * w + 1, J = 2 * w;
    float* mt = w ? m32 : m10;
    clear(acc);
    gemm(acc, blk(I, J), blk(J, J));
    warp_store16(mt, AS_LD, acc, 1.f, lane);
    __syncwarp();
    clear(acc);
    gemm(acc, blk(I, I), mt);
    warp_store16(blk(I, J), AS_LD, acc, -1.f, lane);
    final_block(acc, -1.f, I, J);
  } else if (w < 6) {  // A20 T00, A30 T00, A21 T11, A31 T11
    const int I = 2 + (w & 1), J = (w - 2) >> 1;
    clear(acc);
    gemm(acc, blk(I, J), blk(J, J));
    warp_store16(w == 2 ? x20 : w == 3 ? x30 : w == 4 ? x21 : x31, AS_LD, acc, 1.f, lane);
  } else {  // the diagonal blocks of T diag(beta)
    const int b0 = 2 * (w - 6);
    warp_load16(acc, blk(b0, b0), AS_LD, lane);
    final_block(acc, 1.f, b0, b0);
    warp_load16(acc, blk(b0 + 1, b0 + 1), AS_LD, lane);
    final_block(acc, 1.f, b0 + 1, b0 + 1);
  }
  if (w >= 2) {  // blocks above the diagonal: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
    const int zi = w - 2;
    const int I = zi < 3 ? 0 : zi < 5 ? 1 : 2, J = zi < 3 ? zi + 1 : zi < 5 ? zi - 1 : 3;
    zero_block16(Tt, I, J, lane);
    if (kPrecise) zero_block16(Tlo, I, J, lane);
  }
  if (w == 7) idle();
  sync();
  // ---- level 2
  if (w < 2) {  // X20 = A20 T00 + A21 T10 (w = 0), X30 = A30 T00 + A31 T10 (w = 1)
    float* xp = w ? x30 : x20;
    warp_load16(acc, xp, AS_LD, lane);
    gemm(acc, blk(2 + w, 1), blk(1, 0));
    warp_store16(xp, AS_LD, acc, 1.f, lane);
  } else if (w == 2) {  // T21 = -T22 X21
    clear(acc);
    gemm(acc, blk(2, 2), x21);
    final_block(acc, -1.f, 2, 1);
  } else if (w == 3) {  // T31 = -(T32 X21 + T33 X31)
    clear(acc);
    gemm(acc, blk(3, 2), x21);
    gemm(acc, blk(3, 3), x31);
    final_block(acc, -1.f, 3, 1);
  }
  sync();
  // ---- level 3
  if (w == 4) {  // T20 = -T22 X20
    clear(acc);
    gemm(acc, blk(2, 2), x20);
    final_block(acc, -1.f, 2, 0);
  } else if (w == 5) {  // T30 = -(T32 X20 + T33 X30)
    clear(acc);
    gemm(acc, blk(3, 2), x20);
    gemm(acc, blk(3, 3), x30);
    final_block(acc, -1.f, 3, 0);
  }
}

// The solve of a chunk with near-parallel keys (some |A_rj| >= kSolveAccurateA):
// solve_t_beta<true>.
template <typename Sync, typename Idle>
__device__ __forceinline__ void solve_t_beta_precise(float* As, const float* s_beta, uint8_t* Tt, uint8_t* Tlo, int t,
                                                  int w, int lane, Sync sync, Idle idle) {
  solve_t_beta<true>(As, s_beta, Tt, Tlo, t, w, lane, sync, idle);
}

// Phase 6 epilogue: TMEM columns [tm, tm + 64) = W^T, [tm + 64, tm + 128) = U^T
// (lane = channel) to bf16 K-major rows of the image staging area.  Eight
// warps, arguments as for scatter_single_ref.
__device__ __forceinline__ void stage_w_u(uint32_t tm, uint8_t* stage, int warp, int w8, int lane) {
  const int qd = warp & 3, ch = w8 >> 2;
  const int row = 32 * qd + lane;  // dk channel (W^T) or dv channel (U^T)
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float x[32];
    const uint32_t ta = tm + ((uint32_t)(32 * qd) << 16) + 64 * ch + 32 * hh;
    ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
    ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
    ptx::tmem_wait_ld();
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      const uint4 pk = pack8(x + 8 * k8);
      const uint32_t off = ptx::sw128_chunk(row, 4 * hh + k8);
      *reinterpret_cast<uint4*>(stage + (ch == 0 ? IMG_A1 : IMG_U) + off) = pk;
    }
  }
}

// kGate (GateMode): what the gate argument holds -- log alpha per key channel
// (KDA) or per token (Gated DeltaNet), or raw per-channel logits in fp32 or
// bf16, in which case q and k rows are also L2-normalised and beta is the
// sigmoid of the given logit.
template <int kGate>
__global__ void __launch_bounds__(256, 2)
    kda_tc_chunk_local_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                              const bf16* __restrict__ v, const void* __restrict__ gate,
                              const float* __restrict__ beta, const int32_t* __restrict__ cu_seqlens,
                              int num_seqs, int T, int H, uint32_t num_items, FastDiv fdH, FastDiv fdC,
                              uint8_t* __restrict__ ws, const uint32_t* __restrict__ item_list,
                              const uint32_t* __restrict__ item_cnt, uint32_t list_cap,
                              const int* __restrict__ chunk_total, int* __restrict__ esc_flag) {
  __shared__ __align__(16) float s_beta[C];
  __shared__ float s_nrm[2][C];  // 1 / |k_r|, 1 / |q_r| (only when the call normalises)
  constexpr bool kPrep = gate_prep(kGate);
  __shared__ __align__(16) float s_Ge[4][D];  // G at the end of each 16-token block
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ uint32_t s_tmem;
  __shared__ long long s_loc_s;
  __shared__ int s_loc_n;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  KDA_ALIGNED_DSMEM(sm, dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rs = (size_t)H * D;  // elements between consecutive tokens
  // an empty item list (the usual case): nothing to set up
  if (item_list && item_cnt[blockIdx.x] == 0) return;
  // packed sequences whose cu_seqlens the chunk-table kernel rejected: no work
  if (cu_seqlens && chunk_total && *chunk_total < 0) return;

  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, 256);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&s_bar, 1);
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  // Persistent: this CTA handles items (chunk * H + head) blockIdx.x, + gridDim.x, ...,
  // or, given an item list, entries [0, item_cnt[b]) of list b = blockIdx.x
  // (capacity list_cap each).  Each processed item completes s_bar twice (parities 0 then 1).
  // item = chunk * H + head; unpacked chunk = sequence * fdC.d + chunk-in-sequence (num_items < 2^31)
  const uint32_t n_iter = item_list ? min(item_cnt[blockIdx.x], list_cap) : num_items;
  for (uint32_t it = item_list ? 0u : blockIdx.x; it < n_iter; it += item_list ? 1u : gridDim.x) {
  const uint32_t item = item_list ? item_list[(size_t)blockIdx.x * list_cap + it] : it;
  const uint32_t ci = fdiv(item, fdH);
  const int h = (int)(item - ci * (uint32_t)H);

  long long s0;
  int Cn;
  if (cu_seqlens) {
    if (warp == 0) {
      long long s = 0;
      int cn = 0;
      const bool ok = locate_chunk_warp(cu_seqlens, num_seqs, (long long)ci, &s, &cn);
      if (lane == 0) {
        s_loc_s = s;
        s_loc_n = ok ? cn : -1;
      }
    }
    __syncthreads();
    s0 = s_loc_s;
    Cn = s_loc_n;
  } else {
    const uint32_t bq = fdiv(ci, fdC);
    const int cc = (int)(ci - bq * fdC.d);
    s0 = (long long)bq * T + (long long)cc * C;
    Cn = min(C, T - cc * C);
  }
  if (Cn <= 0) {  // uniform across the CTA: past the last chunk of a packed batch
    __syncthreads();  // everyone has read s_loc before warp 0 rewrites it
    continue;
  }

  uint8_t* img = ws + ((size_t)ci * H + h) * IMG_BYTES;

  // L2 hint for this CTA's next item (packed-free layout only): its q, k, v, g
  // rows, one 128-byte line per lane.
  if (!cu_seqlens && !item_list && item + gridDim.x < num_items) {
    const uint32_t nb = item + gridDim.x;
    const uint32_t nci = fdiv(nb, fdH);
    const int nh = (int)(nb - nci * (uint32_t)H);
    const uint32_t nbq = fdiv(nci, fdC);
    const int ncc = (int)(nci - nbq * fdC.d);
    const long long ns = (long long)nbq * T + (long long)ncc * C;
    const int ncn = min(C, T - ncc * C);
    // 128-byte lines per row: k, q, v 2 each, then the gate (fp32 4, bf16 2, per token 0)
    constexpr int lines = kGate == kGateLogTok ? 6 : kGate == kGateLogitBf16 ? 8 : 10;
    for (int idx = tid; idx < lines * C; idx += 256) {
      const int r = idx / lines, l = idx % lines;
      if (r < ncn) {
        const size_t off = ((size_t)(ns + r) * H + nh) * D;
        const void* pp = l < 2 ? (const void*)(k + off + 64 * l)
                       : l < 4 ? (const void*)(q + off + 64 * (l - 2))
                       : l < 6 ? (const void*)(v + off + 64 * (l - 4))
                       : kGate == kGateLogitBf16
                               ? (const void*)(static_cast<const bf16*>(gate) + off + 64 * (l - 6))
                               : (const void*)(static_cast<const float*>(gate) + off + 32 * (l - 6));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(pp));
      }
    }
  }
  if (tid < C) s_beta[tid] = tid < Cn ? beta_of(beta, kGate, (size_t)(s0 + tid) * H + h) : 0.f;

  // ---- 1. loads; cumulative log-decay G (fp32); rows >= Cn contribute g = 0.
  // The k, q, v rows are loaded here, together with g, and parked in TMEM
  // columns (idle until the first MMA) so that their latency overlaps g's.
  const int co = tid & 15, rg = tid >> 4, J = rg >> 2;  // channel octet, row group, 16-token block
  const int c0 = 8 * co;
  const uint32_t kp = co >> 3, ck = co & 7;  // K-panel and 16-byte chunk of the channels
  const size_t base8 = ((size_t)s0 * H + h) * D + c0;
  uint32_t kst[16], qst[16], vst[16];  // [row u][4 words]: 8 bf16 per row
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = 4 * rg + u;
    uint4 kw = make_uint4(0, 0, 0, 0), qw = kw, vw = kw;
    if (r < Cn) {
      const size_t off = base8 + (size_t)r * rs;
      kw = *reinterpret_cast<const uint4*>(k + off);
      qw = *reinterpret_cast<const uint4*>(q + off);
      vw = *reinterpret_cast<const uint4*>(v + off);
    }
    kst[4 * u] = kw.x; kst[4 * u + 1] = kw.y; kst[4 * u + 2] = kw.z; kst[4 * u + 3] = kw.w;
    qst[4 * u] = qw.x; qst[4 * u + 1] = qw.y; qst[4 * u + 2] = qw.z; qst[4 * u + 3] = qw.w;
    vst[4 * u] = vw.x; vst[4 * u + 1] = vw.y; vst[4 * u + 2] = vw.z; vst[4 * u + 3] = vw.w;
  }
  float G[4][8];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = 4 * rg + u;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (r < Cn) {
      if constexpr (kGate == kGateLogTok) {  // one gate per token, the same on every channel
        const float x = static_cast<const float*>(gate)[(size_t)(s0 + r) * H + h];
        a = make_float4(x, x, x, x);
        b = a;
      } else if constexpr (kGate == kGateLogitBf16) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(static_cast<const bf16*>(gate) + base8 + (size_t)r * rs), x);
        a = make_float4(neg_softplus_sfu(x[0]), neg_softplus_sfu(x[1]), neg_softplus_sfu(x[2]), neg_softplus_sfu(x[3]));
        b = make_float4(neg_softplus_sfu(x[4]), neg_softplus_sfu(x[5]), neg_softplus_sfu(x[6]), neg_softplus_sfu(x[7]));
      } else {
        const float4* gp = reinterpret_cast<const float4*>(static_cast<const float*>(gate) + base8 + (size_t)r * rs);
        a = gp[0];
        b = gp[1];
        if constexpr (kGate == kGateLogitF32) {
          a = make_float4(neg_softplus_sfu(a.x), neg_softplus_sfu(a.y), neg_softplus_sfu(a.z), neg_softplus_sfu(a.w));
          b = make_float4(neg_softplus_sfu(b.x), neg_softplus_sfu(b.y), neg_softplus_sfu(b.z), neg_softplus_sfu(b.w));
        }
      }
    }
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) G[u][e] = (u ? G[u - 1][e] : 0.f) + x[e];
  }
  if constexpr (kPrep) {  // 1 / |k_r| and 1 / |q_r| over dk: the 16 lanes of a half-warp share a row
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float kx[8], qx[8];
      unpack8(make_uint4(kst[4 * u], kst[4 * u + 1], kst[4 * u + 2], kst[4 * u + 3]), kx);
      unpack8(make_uint4(qst[4 * u], qst[4 * u + 1], qst[4 * u + 2], qst[4 * u + 3]), qx);
      float sk = 0.f, sq = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sk = fmaf(kx[e], kx[e], sk);
        sq = fmaf(qx[e], qx[e], sq);
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
      }
      if (co == 0) {
        s_nrm[0][4 * rg + u] = rsqrtf(fmaxf(sk, 1e-24f));
        s_nrm[1][4 * rg + u] = rsqrtf(fmaxf(sq, 1e-24f));
      }
    }
  }
  float* s_tot = reinterpret_cast<float*>(sm + KA_XK);  // [16][128] row-group totals (XK is built later)
  reinterpret_cast<float4*>(s_tot + rg * D + c0)[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
  reinterpret_cast<float4*>(s_tot + rg * D + c0)[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // stash: warp w uses lanes 32 (w mod 4) .., columns 48 (w / 4) + [k 0..15 | q 16..31 | v 32..47]
  const uint32_t stash = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 48 * (warp >> 2);
  ptx::tmem_st16u(stash, kst);
  ptx::tmem_st16u(stash + 16, qst);
  ptx::tmem_st16u(stash + 32, vst);
  ptx::tmem_wait_st();
  {
    float off[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q2 = 0; q2 < 15; ++q2) {
      if (q2 < rg) {
        const float4 t0 = reinterpret_cast<const float4*>(s_tot + q2 * D + c0)[0];
        const float4 t1 = reinterpret_cast<const float4*>(s_tot + q2 * D + c0)[1];
        off[0] += t0.x; off[1] += t0.y; off[2] += t0.z; off[3] += t0.w;
        off[4] += t1.x; off[5] += t1.y; off[6] += t1.z; off[7] += t1.w;
      }
    }
    if constexpr (kGate == kGateLogTok) {  // one gate per token: every channel has the same G
#pragma unroll
      for (int e = 1; e < 8; ++e) off[e] = off[0];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) G[u][e] += off[e];
  }
  bool steep = false;  // some channel decays below the single-reference range
  if ((rg & 3) == 3) {
    reinterpret_cast<float4*>(&s_Ge[J][c0])[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
    reinterpret_cast<float4*>(&s_Ge[J][c0])[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
#pragma unroll
    for (int e = 0; e < 8; ++e) steep |= (J == 3) && !(G[3][e] >= kChunkRefMinG);
  }
  // The previous item's image bulk store has read its staging area before the
  // builder below overwrites it.
  if (tid == 0) ptx::bulk_wait_read0();
  // G is non-increasing (g <= 0), so G at the chunk's last row is each channel's minimum.
  const bool fast = !__syncthreads_or(steep);

  // ---- 2. decay-scaled bf16 operands, 16-byte stores
  uint32_t qgp[2][8];  // Q o e^G of this thread's 4 tokens, bf16 pairs per channel
  if (fast) {
    // Single reference (chunk start): a = e^{G} <= 1, rho = e^{-G} >= 1.
    float gam[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) gam[e] = __expf(s_Ge[3][c0 + e]);
    float qg_prev[8];
    uint8_t* l3 = sm + KA_L3 + kp * 16384;
    uint8_t* rb = sm + KA_RB + kp * 20480;
#pragma unroll
    for (int up = 0; up < 2; ++up) {  // two rows per TMEM round trip
      uint32_t kr2[2][4], qr2[2][4], vr2[2][4];
#pragma unroll
      for (int uu = 0; uu < 2; ++uu) {
        ptx::tmem_ld4u(stash + 4 * (2 * up + uu), kr2[uu]);
        ptx::tmem_ld4u(stash + 16 + 4 * (2 * up + uu), qr2[uu]);
        ptx::tmem_ld4u(stash + 32 + 4 * (2 * up + uu), vr2[uu]);
      }
      ptx::tmem_wait_ld();
#pragma unroll
      for (int uu = 0; uu < 2; ++uu) {
      const int u = 2 * up + uu, r = 4 * rg + u;
      const uint32_t* kr4 = kr2[uu];
      const uint32_t* qr4 = qr2[uu];
      const uint32_t* vr4 = vr2[uu];
      float kv[8], qv[8];
      unpack8(make_uint4(kr4[0], kr4[1], kr4[2], kr4[3]), kv);
      unpack8(make_uint4(qr4[0], qr4[1], qr4[2], qr4[3]), qv);
      if constexpr (kPrep) normalise_rows(kv, qv, s_nrm[0][r], s_nrm[1][r]);
      float o_ka[8], o_qa[8], o_kr[8], o_kb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = G[u][e] * 1.4426950408889634f;  // G log2(e), in [-115.5, 0]
        const float a = ptx::ex2(t);     // e^G in (0, 1]
        const float rho = ptx::ex2(-t);  // e^-G in [1, e^80]
        o_ka[e] = kv[e] * a;
        o_qa[e] = qv[e] * a;
        o_kr[e] = kv[e] * rho;
        o_kb[e] = o_kr[e] * gam[e];          // K o e^{G_last - G}
        if (u & 1) qgp[u >> 1][e] = ptx::pack_bf16x2(qg_prev[e], o_qa[e]);
        else qg_prev[e] = o_qa[e];
      }
      *reinterpret_cast<uint4*>(l3 + ptx::sw128_chunk(r, ck)) = pack8(o_ka);
      *reinterpret_cast<uint4*>(l3 + ptx::sw128_chunk(64 + r, ck)) = pack8(o_qa);
      *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(r, ck)) = pack8(o_kr);
      *reinterpret_cast<uint4*>(img + IMG_KB + kp * 8192 + ptx::sw128_chunk(r, ck)) = pack8(o_kb);
      *reinterpret_cast<uint4*>(sm + KA_BV + kp * 8192 + ptx::sw128_chunk(r, ck)) =
          make_uint4(vr4[0], vr4[1], vr4[2], vr4[3]);
      }
    }
  } else {
    float Gb[8], GeJ[8], eGb[8], invD[8], lam[8], sig1[8], sig2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = c0 + e;
      GeJ[e] = s_Ge[J][c];
      Gb[e] = J ? s_Ge[J - 1][c] : 0.f;
      eGb[e] = __expf(Gb[e]);                        // e^{G} at the block start
      invD[e] = __expf(Gb[e] - GeJ[e]);              // 1 / (block decay), >= 1
      lam[e] = __expf(s_Ge[3][c] - GeJ[e]);          // block end -> chunk end
      sig1[e] = J <= 1 ? __expf(s_Ge[J + 1][c] - GeJ[e]) : 0.f;  // for row block J + 2
      sig2[e] = J == 0 ? __expf(s_Ge[2][c] - GeJ[e]) : 0.f;      // for row block 3
    }
    float qg_prev[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = 4 * rg + u, e16 = r & 15;
      uint32_t kr4[4], qr4[4], vr4[4];
      ptx::tmem_ld4u(stash + 4 * u, kr4);
      ptx::tmem_ld4u(stash + 16 + 4 * u, qr4);
      ptx::tmem_ld4u(stash + 32 + 4 * u, vr4);
      ptx::tmem_wait_ld();
      const uint4 kw = make_uint4(kr4[0], kr4[1], kr4[2], kr4[3]);
      const uint4 qw = make_uint4(qr4[0], qr4[1], qr4[2], qr4[3]);
      const uint4 vw = make_uint4(vr4[0], vr4[1], vr4[2], vr4[3]);
      float kv[8], qv[8];
      unpack8(kw, kv);
      unpack8(qw, qv);
      if constexpr (kPrep) normalise_rows(kv, qv, s_nrm[0][r], s_nrm[1][r]);
      float o_lk[8], o_lq[8], o_r0[8], o_r1[8], o_r2[8], o_rd[8], o_kb[8], o_xk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = __expf(G[u][e] - Gb[e]);   // (0, 1]
        const float b = __expf(GeJ[e] - G[u][e]);  // (0, 1]
        const float ka = kv[e] * a, kb = kv[e] * b;
        o_lk[e] = ka;
        o_lq[e] = qv[e] * a;
        // Q o e^G for the state pass, packed over token pairs (u, u+1)
        const float qg = o_lq[e] * eGb[e];
        if (u & 1) qgp[u >> 1][e] = ptx::pack_bf16x2(qg_prev[e], qg);
        else qg_prev[e] = qg;
        o_r0[e] = kb;
        o_r1[e] = kb * sig1[e];
        o_r2[e] = kb * sig2[e];
        o_rd[e] = kb * invD[e];
        o_kb[e] = kb * lam[e];
        o_xk[e] = ka * eGb[e];
      }
      uint8_t* l3 = sm + KA_L3 + kp * 16384;
      uint8_t* rb = sm + KA_RB + kp * 20480;
      *reinterpret_cast<uint4*>(l3 + ptx::sw128_chunk(r, ck)) = pack8(o_lk);
      *reinterpret_cast<uint4*>(l3 + ptx::sw128_chunk(64 + r, ck)) = pack8(o_lq);
      // right operands: rows 16 (I (I - 1) / 2 + J) + e16 for row block I = J+1..3; diagonal at 96 + r
      if (J <= 2) *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(16 * ((J + 1) * J / 2 + J) + e16, ck)) = pack8(o_r0);
      if (J <= 1) *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(16 * ((J + 2) * (J + 1) / 2 + J) + e16, ck)) = pack8(o_r1);
      if (J == 0) *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(48 + e16, ck)) = pack8(o_r2);
      *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(96 + r, ck)) = pack8(o_rd);
      // Kbar = K o e^{G_last - G} (image, MN-major panel = channel / 64, row = token)
      *reinterpret_cast<uint4*>(img + IMG_KB + kp * 8192 + ptx::sw128_chunk(r, ck)) = pack8(o_kb);
      // K o e^G and V: MN-major A operands of the WY products (beta is folded into T)
      *reinterpret_cast<uint4*>(sm + KA_XK + kp * 8192 + ptx::sw128_chunk(r, ck)) = pack8(o_xk);
      *reinterpret_cast<uint4*>(sm + KA_BV + kp * 8192 + ptx::sw128_chunk(r, ck)) = vw;
    }
  }
  {
    // Q o e^G into the lower panel of the [W; Q e^G] image (MN-major, row = channel,
    // 64 tokens per 128-byte row): this thread's 4 tokens are 8 contiguous bytes
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = c0 + e;
      *reinterpret_cast<uint2*>(img + IMG_A1 + 16384 + c * 128 + ((((4 * rg) >> 3) ^ c) & 7) * 16 +
                                8 * (rg & 1)) = make_uint2(qgp[0][e], qgp[1][e]);
    }
  }
  if (rg == 0) {
    float gm[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) gm[e] = expf(s_Ge[3][c0 + e]);
    reinterpret_cast<float4*>(img + IMG_G)[2 * co] = make_float4(gm[0], gm[1], gm[2], gm[3]);
    reinterpret_cast<float4*>(img + IMG_G)[2 * co + 1] = make_float4(gm[4], gm[5], gm[6], gm[7]);
  }

  // ---- 3. [A'; P'] = [K a; Q a] (right operands)^T : M=128, K=128,
  //         N=64 (single reference) or 160 (block references)
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    ptx::tc_fence_after();
    const uint32_t id = fast ? ptx::idesc_bf16(128, 64, false, false) : ptx::idesc_bf16(128, 160, false, false);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t ad = ptx::sdesc_sw128(sb + KA_L3 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = ptx::sdesc_sw128(sb + KA_RB + (kk >> 2) * 20480 + (kk & 3) * 32, 16, 1024);
      ptx::mma_bf16(tmem, ad, bd, id, kk > 0);
    }
    ptx::mma_commit(&s_bar);
  }
  ptx::mbar_wait_bounded(&s_bar, 0);  // first completion of this item
  ptx::tc_fence_after();

  // ---- 4. scatter A (fp32, beta-scaled) and P (bf16, lower incl. diagonal, zero above)
  bool big = false;  // some |A_rj| this thread wrote >= kSolveAccurateA
  if (fast) {  // TMEM columns 0..63 hold whole rows
    big = scatter_single_ref(tmem, s_beta, reinterpret_cast<float*>(sm + KA_AS), sm + KA_PT, warp, warp, lane);
  } else {
    const int qd = warp & 3, ch = warp >> 2;
    const int rho = 32 * qd + lane;
    const bool isK = rho < 64;
    const int r = rho & 63, I = r >> 4;
    const float br = s_beta[r];
    float* As = reinterpret_cast<float*>(sm + KA_AS);
    float xs[5][16];
#pragma unroll
    for (int grp = 0; grp < 5; ++grp)
      ptx::tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + 80 * ch + 16 * grp, xs[grp]);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int grp = 0; grp < 5; ++grp) {
      const int col0 = 80 * ch + 16 * grp;
      float* x = xs[grp];
      const bool diag = col0 >= 96;
      int Jb;
      bool use;
      if (!diag) {
        const int seg = col0 >> 4;
        const int Is = seg == 0 ? 1 : (seg < 3 ? 2 : 3);
        Jb = seg - Is * (Is - 1) / 2;
        use = Is == I;
      } else {
        Jb = (col0 - 96) >> 4;
        use = Jb == I;
      }
      if (isK) {
        if (use) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            x[e] = (!diag || 16 * Jb + e < r) ? br * x[e] : 0.f;
            big |= fabsf(x[e]) >= kSolveAccurateA;
          }
          float4* dst = reinterpret_cast<float4*>(As + r * AS_LD + 16 * Jb);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_float4(x[4 * v4], x[4 * v4 + 1], x[4 * v4 + 2], x[4 * v4 + 3]);
        }
      } else if (use || (diag && Jb > I)) {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = (!diag || (Jb == I && 16 * Jb + e <= r)) ? x[e] : 0.f;
        *reinterpret_cast<uint4*>(sm + KA_PT + ptx::sw128_chunk(r, 2 * Jb)) = pack8(x);
        *reinterpret_cast<uint4*>(sm + KA_PT + ptx::sw128_chunk(r, 2 * Jb + 1)) = pack8(x + 8);
      }
    }
  }
  ptx::tc_fence_before();
  // near-parallel keys: this call's result is recomputed by the single-pass
  // kernel in its precise form (launch_chunk_tc)
  if (__syncthreads_or(big) && tid == 0) *esc_flag = 1;

  // ---- 5. T = (I + A)^{-1} and T diag(beta) in bf16
  solve_t_beta<false>(reinterpret_cast<float*>(sm + KA_AS), s_beta, sm + KA_TT, nullptr, tid, warp, lane,
                      [] { __syncthreads(); }, [] {});

  // ---- 6. W^T = (K e^G)^T (T diag(beta))^T, U^T = V^T (T diag(beta))^T : M=128, N=64, K=64
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t bd = ptx::sdesc_sw128(sb + KA_TT + kk * 32, 16, 1024);
      // K o e^G: the K part of L3 (panel stride 16 KB) on the single-reference path
      const uint64_t xd = fast ? ptx::sdesc_sw128(sb + KA_L3 + kk * 2048, 16384, 1024)
                               : ptx::sdesc_sw128(sb + KA_XK + kk * 2048, 8192, 1024);
      ptx::mma_bf16(tmem + 0, xd, bd, id, kk > 0);
      ptx::mma_bf16(tmem + 64, ptx::sdesc_sw128(sb + KA_BV + kk * 2048, 8192, 1024), bd, id, kk > 0);
    }
    ptx::mma_commit(&s_bar);
  }
  ptx::mbar_wait_bounded(&s_bar, 1);  // second completion of this item
  ptx::tc_fence_after();
  stage_w_u(tmem, sm + KA_IMG_STAGE, warp, warp, lane);

  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();  // every TMEM read of this item is done before the next item's stash
  if (tid == 0) {
    ptx::bulk_s2g(img + IMG_P, sm + KA_IMG_STAGE, IMG_A1 + 16384 - IMG_P);
    ptx::bulk_commit();
  }
  }  // item loop
  if (tid == 0) ptx::bulk_wait0();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// Kernel 2: the state pass.  Persistent; CTA b handles units b, b + grid, ...
// Thread t: state row c = 32 (warp mod 4) + lane, columns 64 (warp / 4) + [0, 64).
// ---------------------------------------------------------------------------
// State-pass passes.  A sequence split into segments of L chunks: the map
// pass runs, for every segment but the last, the linear part M (state from I,
// no U term) and the offset N (state from 0) of the segment's affine map
// S -> M S + N; the combine kernel chains S0 through the maps; the final pass
// runs every segment from its entry state and writes the outputs.
constexpr int kPassPlain = 0, kPassMaps = 1, kPassFinal = 2;

// Entry states of the segments: S_{p+1} = M_p S_p + N_p, in fp32.  One CTA per
// (unit, 8-column block); thread t owns row t / 2, columns 4 (t mod 2) .. + 3.
__global__ void __launch_bounds__(256)
    kda_tc_seg_combine_kernel(const float* __restrict__ maps, const float* __restrict__ S0,
                              float* __restrict__ seg_init, int P, const int* __restrict__ esc_flag) {
  if (*esc_flag) return;  // the single-pass kernel recomputes the call
  __shared__ __align__(16) float Ss[D][8];
  const long long u = blockIdx.x / (D / 8);
  const int j0 = (blockIdx.x % (D / 8)) * 8;
  const int tid = threadIdx.x, c = tid >> 1, jq = 4 * (tid & 1);
  float4 cur = S0 ? *reinterpret_cast<const float4*>(S0 + ((size_t)u * D + c) * D + j0 + jq)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  *reinterpret_cast<float4*>(&Ss[c][jq]) = cur;
  // segment 0's entry state is S0 itself; the final pass reads this copy, so
  // that an S_out aliasing S0 may be written while other segments still run
  *reinterpret_cast<float4*>(seg_init + ((size_t)(u * P) * D + c) * D + j0 + jq) = cur;
  __syncthreads();
  for (int p = 0; p + 1 < P; ++p) {
    const float* Nm = maps + (size_t)((u * (P - 1) + p) * 2) * D * D;
    const float* Mrow = Nm + (size_t)D * D + (size_t)c * D;
    float4 acc = *reinterpret_cast<const float4*>(Nm + (size_t)c * D + j0 + jq);
#pragma unroll 4
    for (int k4 = 0; k4 < D / 4; ++k4) {
      const float4 m = reinterpret_cast<const float4*>(Mrow)[k4];
      const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 sv = *reinterpret_cast<const float4*>(&Ss[4 * k4 + e][jq]);
        acc = f4_fma(mk[e], sv, acc);
      }
    }
    __syncthreads();  // every read of the old state is done
    *reinterpret_cast<float4*>(&Ss[c][jq]) = acc;
    *reinterpret_cast<float4*>(seg_init + ((size_t)(u * P + p + 1) * D + c) * D + j0 + jq) = acc;
    __syncthreads();
  }
}


__global__ void __launch_bounds__(256, 2)
    kda_tc_state_pass_kernel(const uint8_t* __restrict__ ws, const float* __restrict__ S0,
                             float* __restrict__ S_out, bf16* __restrict__ o,
                             const int32_t* __restrict__ cu_seqlens, int N, int T, int H,
                             int seg_chunks, int pass, float* __restrict__ maps,
                             const float* __restrict__ seg_init, const int* __restrict__ chunk_total,
                             const int* __restrict__ esc_flag) {
  __shared__ __align__(8) uint64_t s_full[3];  // image parts: 0 [W; Q e^G], 1 U^T, 2 P + Kbar + gamma
  __shared__ __align__(8) uint64_t s_mma1, s_mma2;
  __shared__ uint32_t s_tmem;
  __shared__ long long s_u_first, s_u_start;
  __shared__ int s_u_len;
  __shared__ int s_abort;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  KDA_ALIGNED_DSMEM(sm, dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);

  // packed sequences whose cu_seqlens the chunk-table kernel rejected: the
  // outputs are left untouched
  if (cu_seqlens && chunk_total && *chunk_total < 0) return;
  // a chunk with near-parallel keys: the single-pass kernel recomputes the call
  if (*esc_flag) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, ch = warp >> 2;
  const int c = 32 * qd + lane;  // state row; rows 0..63 of X are tokens (-E), 64..127 outputs
  const uint32_t lane_off = (uint32_t)(32 * qd) << 16;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) ptx::mbar_init(&s_full[i], 1);
    ptx::mbar_init(&s_mma1, 1);
    ptx::mbar_init(&s_mma2, 1);
    ptx::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // TMEM: X (columns 0..127) and the fp32 state S (columns 128..255), lane = row.
  const uint32_t tX = s_tmem, tS = s_tmem + 128;
  const uint32_t tXr = tX + lane_off + 64 * ch, tSr = tS + lane_off + 64 * ch;

  uint32_t it = 0;  // chunks processed by this CTA: every barrier completes once per chunk
  bool pend[3] = {false, false, false};  // (thread 0) a load in flight not yet waited for
  const long long units = (long long)N * H;
  const long long ncps = (T + C - 1) / C;
  const int P = seg_chunks > 0 ? (int)((ncps + seg_chunks - 1) / seg_chunks) : 1;
  const long long items = pass == kPassMaps ? units * (P - 1) * 2 : units * P;
  bool aborted = false;
  for (long long item = blockIdx.x; item < items && !aborted; item += gridDim.x) {
    // kind 1: the linear part M of a segment's map (state from I, no U term);
    // kind 0: its offset N (state from 0), or an ordinary run.
    long long u;
    int p = 0, kind = 0;
    if (pass == kPassMaps) {
      kind = (int)(item & 1);
      const long long r = item >> 1;
      p = (int)(r % (P - 1));
      u = r / (P - 1);
    } else {
      p = (int)(item % P);
      u = item / P;
    }
    const int n = (int)(u / H), h = (int)(u % H);
    long long first, start;
    int len;
    if (seg_chunks > 0) {
      first = (long long)n * ncps + (long long)p * seg_chunks;
      start = (long long)n * T + (long long)p * seg_chunks * C;
      len = (int)min((long long)seg_chunks * C, (long long)T - (long long)p * seg_chunks * C);
    } else if (cu_seqlens) {
      if (warp == 0) {
        const long long f = chunks_before_warp(cu_seqlens, n);
        if (lane == 0) {
          long long t0, t1;
          checked_seq_range(cu_seqlens, n, T, &t0, &t1);  // T = total tokens when packed
          // the unit's images must lie inside the workspace (T / C + N chunks)
          const bool in_ws = f >= 0 && f + (t1 - t0 + C - 1) / C <= (long long)T / C + N;
          if (!in_ws) raise_device_error(kDevErrBadSeqlens);
          s_u_first = in_ws ? f : 0;
          s_u_start = t0;
          s_u_len = in_ws ? (int)(t1 - t0) : 0;
        }
      }
      __syncthreads();
      first = s_u_first;
      start = s_u_start;
      len = s_u_len;
      __syncthreads();  // read before warp 0 rewrites them for the next item
    } else {
      first = (long long)n * ncps;
      start = (long long)n * T;
      len = T;
    }
    const int nc = (len + C - 1) / C;
    const size_t soff = ((size_t)u * D + c) * D + 64 * ch;
    const float* S_src = nullptr;
    if (pass == kPassFinal)  // every segment's entry state, segment 0's included (a copy of S0)
      S_src = seg_init + ((size_t)(u * P + p) * D + c) * D + 64 * ch;
    else if (pass != kPassMaps && S0)
      S_src = S0 + soff;
    const bool no_u = pass == kPassMaps && kind == 1;

    // initial state: fp32 into TMEM, bf16 into the MMA operand
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      float x[16];
      if (S_src) {
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const float4 t = reinterpret_cast<const float4*>(S_src)[4 * q4 + j4];
          x[4 * j4] = t.x; x[4 * j4 + 1] = t.y; x[4 * j4 + 2] = t.z; x[4 * j4 + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = (no_u && 64 * ch + 16 * q4 + e == c) ? 1.f : 0.f;
      }
      ptx::tmem_st16(tSr + 16 * q4, x);
#pragma unroll
      for (int k8 = 0; k8 < 2; ++k8)
        *reinterpret_cast<uint4*>(sm + KB_SB + ch * 16384 + ptx::sw128_chunk(c, 2 * q4 + k8)) = pack8(x + 8 * k8);
    }
    ptx::tmem_wait_st();
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();

    auto img_of = [&](long long chunk_idx) { return ws + ((size_t)chunk_idx * H + h) * IMG_BYTES; };
    auto load_wq = [&](long long ci) {
      ptx::mbar_arrive_expect_tx(&s_full[0], 32768);
      ptx::bulk_g2s(sm + KB_WQ, img_of(ci) + IMG_A1, 32768, &s_full[0]);
      pend[0] = true;
    };
    auto load_ue_pk = [&](long long ci) {
      ptx::mbar_arrive_expect_tx(&s_full[1], 16384);
      ptx::bulk_g2s(sm + KB_UE, img_of(ci) + IMG_U, 16384, &s_full[1]);
      ptx::mbar_arrive_expect_tx(&s_full[2], 8192 + 16896);
      ptx::bulk_g2s(sm + KB_P, img_of(ci) + IMG_P, 8192, &s_full[2]);
      ptx::bulk_g2s(sm + KB_KG, img_of(ci) + IMG_KB, 16896, &s_full[2]);
      pend[1] = pend[2] = true;
    };
    if (tid == 0 && nc > 0) {
      load_wq(first);
      load_ue_pk(first);
    }
    for (int cc = 0; cc < nc; ++cc, ++it) {
      const uint32_t ph = it & 1;
      const long long s = start + (long long)cc * C;
      const int Cn = min(C, len - cc * C);
      // ---- X = [W; Q e^G] S_bf16  (M=128, N=128, K=128, both MN-major)
      if (tid == 0) {
        if (!ptx::mbar_wait_bounded(&s_full[0], ph)) s_abort = 1;
        pend[0] = false;
        ptx::tc_fence_after();
        constexpr uint32_t id1 = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16(tX, ptx::sdesc_sw128(sb + KB_WQ + kk * 2048, 16384, 1024),
                        ptx::sdesc_sw128(sb + KB_SB + kk * 2048, 16384, 1024), id1, kk > 0);
        ptx::mma_commit(&s_mma1);
      }
      if (!ptx::mbar_wait_bounded(&s_full[1], ph)) s_abort = 1;
      if (!ptx::mbar_wait_bounded(&s_full[2], ph)) s_abort = 1;
      // gamma o S in TMEM (the state pass's decay), while the MMA runs
      const float gam = reinterpret_cast<const float*>(sm + KB_KG + 16384)[c];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float x[16];
        ptx::tmem_ld16(tSr + 16 * q4, x);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] *= gam;
        ptx::tmem_st16(tSr + 16 * q4, x);
      }
      if (!ptx::mbar_wait_bounded(&s_mma1, ph)) s_abort = 1;
      ptx::tc_fence_after();
      // E = U - W S for this thread's token row (rows 0..63 of X hold W S); U
      // from U^T[dv][j]: a warp reads 32 tokens of one dv row per load.
      uint32_t e_pk[32];
      if (qd < 2) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[32];
          ptx::tmem_ld16(tXr + 32 * hh, *reinterpret_cast<float(*)[16]>(x));
          ptx::tmem_ld16(tXr + 32 * hh + 16, *reinterpret_cast<float(*)[16]>(x + 16));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int dv = 64 * ch + 32 * hh + 2 * e;
            float u0 = 0.f, u1 = 0.f;
            if (!no_u) {
              u0 = __bfloat162float(*reinterpret_cast<const bf16*>(sm + KB_UE + ptx::sw128(dv, c)));
              u1 = __bfloat162float(*reinterpret_cast<const bf16*>(sm + KB_UE + ptx::sw128(dv + 1, c)));
            }
            e_pk[16 * hh + e] = ptx::pack_bf16x2(u0 - x[2 * e], u1 - x[2 * e + 1]);
          }
        }
      }
      ptx::tmem_wait_st();
      __syncthreads();  // every read of U^T is done before E overwrites it
      if (tid == 0 && cc + 1 < nc) load_wq(first + cc + 1);  // the first MMA has read [W; Q e^G]
      if (qd < 2) {
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8)
          *reinterpret_cast<uint4*>(sm + KB_UE + ch * 8192 + ptx::sw128_chunk(c, k8)) =
              make_uint4(e_pk[4 * k8], e_pk[4 * k8 + 1], e_pk[4 * k8 + 2], e_pk[4 * k8 + 3]);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        ptx::tc_fence_after();
        // S += Kbar^T E  (M=128, N=128, K=64, both MN-major), onto gamma o S
        constexpr uint32_t id2 = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tS, ptx::sdesc_sw128(sb + KB_KG + kk * 2048, 8192, 1024),
                        ptx::sdesc_sw128(sb + KB_UE + kk * 2048, 8192, 1024), id2, 1);
        // X += [*; P] E: rows 64..127 become O = Q e^G S + P E (rows 0..63 are dead).
        // The map pass writes no output.
        constexpr uint32_t id3 = ptx::idesc_bf16(128, 128, false, true);
        if (pass != kPassMaps) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16(tX, ptx::sdesc_sw128(sb + KB_P - 8192 + kk * 32, 16, 1024),
                          ptx::sdesc_sw128(sb + KB_UE + kk * 2048, 8192, 1024), id3, 1);
        }
        ptx::mma_commit(&s_mma2);
      }
      if (!ptx::mbar_wait_bounded(&s_mma2, ph)) s_abort = 1;
      ptx::tc_fence_after();
      if (tid == 0) {  // U^T / E, P, Kbar and gamma are all read
        pend[1] = pend[2] = false;
        if (cc + 1 < nc) load_ue_pk(first + cc + 1);
      }
      // the state operand of the next chunk
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float x[16];
        ptx::tmem_ld16(tSr + 16 * q4, x);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int k8 = 0; k8 < 2; ++k8)
          *reinterpret_cast<uint4*>(sm + KB_SB + ch * 16384 + ptx::sw128_chunk(c, 2 * q4 + k8)) = pack8(x + 8 * k8);
      }
      // rows 64..127 of X: the chunk's outputs
      if (qd >= 2 && pass != kPassMaps) {
        const int r = c - 64;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[32];
          ptx::tmem_ld16(tXr + 32 * hh, *reinterpret_cast<float(*)[16]>(x));
          ptx::tmem_ld16(tXr + 32 * hh + 16, *reinterpret_cast<float(*)[16]>(x + 16));
          ptx::tmem_wait_ld();
          if (r < Cn) {
            bf16* dst = o + ((size_t)(s + r) * H + h) * D + 64 * ch + 32 * hh;
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) reinterpret_cast<uint4*>(dst)[k8] = pack8(x + 8 * k8);
          }
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (s_abort) {
        aborted = true;
        break;
      }
    }
    float* S_dst = nullptr;
    if (pass == kPassMaps)
      S_dst = maps + ((size_t)((u * (P - 1) + p) * 2 + kind) * D + c) * D + 64 * ch;
    else if (S_out && p == P - 1)
      S_dst = S_out + soff;
    if (!aborted && S_dst) {
      ptx::tc_fence_after();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float x[16];
        ptx::tmem_ld16(tSr + 16 * q4, x);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4)
          reinterpret_cast<float4*>(S_dst)[4 * q4 + j4] = make_float4(x[4 * j4], x[4 * j4 + 1], x[4 * j4 + 2], x[4 * j4 + 3]);
      }
    }
    ptx::tc_fence_before();
    __syncthreads();  // TMEM S of this item is read before the next item overwrites it
  }
  // copies still in flight after an abort must land before shared memory is released
  if (tid == 0 && aborted) {  // they belong to the chunk after the one that gave up
    for (int i = 0; i < 3; ++i)
      if (pend[i]) ptx::mbar_wait_bounded(&s_full[i], (it + 1) & 1);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(s_tmem, 256);
}

}  // namespace tc
}  // namespace kda

#include "kda_chunk_ws.cuh"     // warp-specialised chunk-local kernel
#include "kda_chunk_fused.cuh"  // single-pass kernel

namespace kda {

// Chunks per sequence segment for the state pass, or 0 for none.  Segments
// pay off when the (sequence, head) units are too few to fill the SMs and
// each sequence is long: the serial chain of one unit then bounds the time.
// Model, in chunk-step times: unsegmented ceil(units / sms) * nc; segmented
// (P segments of L chunks) ceil(2 units (P-1) / sms) L for the maps,
// ceil(units P / sms) L for the final pass, plus P for the combine.
// `force` > 0 fixes L, < 0 disables segments; packed layouts are never split.
inline int tc_segment_chunks(int B, int T, int H, int num_seqs, int sms, int force) {
  if (num_seqs > 0 || force < 0 || B <= 0 || T <= 0 || sms <= 0) return 0;
  const long long nc = (T + tc::C - 1) / tc::C;
  if (force > 0) return force < nc ? force : 0;
  const long long units = (long long)B * H;
  if (2 * units > sms || nc < 64) return 0;
  auto waves = [&](long long n) { return (n + sms - 1) / sms; };
  long long best_cost = waves(units) * nc;
  int best_L = 0;
  const long long pmax = std::min<long long>(nc / 16, 8LL * sms / units);
  for (long long P = 2; P <= pmax; ++P) {
    const long long L = (nc + P - 1) / P, Pe = (nc + L - 1) / L;
    const long long cost = waves(2 * units * (Pe - 1)) * L + waves(units * Pe) * L + Pe;
    if (cost < best_cost) {
      best_cost = cost;
      best_L = (int)L;
    }
  }
  return best_L;
}

// Which tensor-core prefill runs: the single-pass kernel (one CTA per SM takes
// whole (sequence, head) units) or the two-kernel path (chunk-local kernel over
// all chunks at once, then the state pass), which alone carries the sequence
// segments that long sequences with too few units for the GPU need.  `force`:
// 0 automatic (the single pass unless segments were chosen), 1 single pass,
// 2 two kernels.  Returns true for the single pass.
constexpr int kPathAuto = 0, kPathFused = 1, kPathTwoKernel = 2;
// Which tensor-core prefill a call runs.  The single pass keeps one
// (sequence, head) unit per SM, so its time goes in whole waves of units; the
// two-kernel path spreads the chunk-local work over every SM.  Measured
// (B200, 148 SMs): B4 H32 T4096 (128 units, one wave) 0.39 against 0.50 ms;
// B8 H32 T8192 (256 units, two waves) 1.63 against 1.70 ms; B16 H32 T8192
// (512 units, four waves) 3.06 against 3.38 ms; B1 H16 T4096 (16 units) 0.34
// against 0.24 ms; 16 packed sequences of 1 K to 64 K tokens, 32 heads: 11.7
// against 15.6 ms (its CTAs take whole units longest first, where the
// two-kernel state pass deals them out in order).  Automatic choice: the
// single pass for packed sequences with at least one unit per SM, and for
// batches whose units fill their waves to 80% or more; the two-kernel path
// otherwise (with sequence segments for few, long sequences).  Both paths
// meet the same tolerance (the two-kernel path through its precise fallback).
inline bool tc_use_fused(int B, int T, int H, int num_seqs, int sms, int seg_chunks, int force) {
  if (force == kPathTwoKernel || seg_chunks > 0 || sms <= 0) return false;
  const long long N = num_seqs > 0 ? num_seqs : B;
  const long long tokens = (long long)B * T;
  if (tokens >= (1LL << 31) || N * H >= (1LL << 31)) return false;
  if (force == kPathFused) return true;
  const long long units = N * H;
  if (num_seqs > 0) return units >= sms;
  const long long waves = (units + sms - 1) / sms;
  return units * 10 >= waves * sms * 8 && (T + tc::C - 1) / tc::C >= 16;
}

// Workspace: the per-chunk images, then (segmented runs) the maps [N | M] of
// every segment but the last and the entry state of every segment, fp32,
// then the warp-specialised kernel's per-CTA item lists (at most
// items + kMaxListCtas entries and kMaxListCtas counts, uint32), then (packed
// sequences) its chunk table, {first token, rows} per chunk, and the count,
// then the precise-fallback flag and the single-pass kernel's own workspace.
constexpr int kMaxListCtas = 1024;
struct TcWorkspace {
  size_t images, maps, seg_init, lists, table, esc, fused, total;
};
inline TcWorkspace tc_workspace_layout(long long max_chunks, int H, long long units, int T, int seg_chunks,
                                       int num_seqs) {
  TcWorkspace w{};
  w.images = (size_t)max_chunks * (size_t)H * tc::IMG_BYTES;
  w.maps = w.seg_init = w.lists = (w.images + 255) & ~(size_t)255;
  if (seg_chunks > 0) {
    const long long nc = (T + tc::C - 1) / tc::C;
    const long long P = (nc + seg_chunks - 1) / seg_chunks;
    const size_t mat = (size_t)tc::D * tc::D * sizeof(float);
    w.seg_init = w.maps + (size_t)units * (size_t)(P - 1) * 2 * mat;
    w.lists = w.seg_init + (size_t)units * (size_t)P * mat;
  }
  w.table = (w.lists + ((size_t)max_chunks * (size_t)H + 2 * kMaxListCtas) * sizeof(uint32_t) + 255) & ~(size_t)255;
  w.esc = (w.table + (size_t)max_chunks * sizeof(int2) + 16 + 255) & ~(size_t)255;
  w.fused = w.esc + 256;
  w.total = w.fused + fu::fused_workspace_bytes(num_seqs, units);
  return w;
}

inline cudaError_t launch_chunk_tc(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                   const __nv_bfloat16* v, const void* g, const float* beta,
                                   const float* S0, __nv_bfloat16* o, float* S_out,
                                   const int32_t* cu_seqlens, int N, int B, int T, int H,
                                   long long max_chunks, void* workspace, int gmode, int seg_chunks,
                                   int local_kernel, cudaEvent_t* ev, cudaStream_t stream) {
  static PerDeviceOnce s_attrs;
  cudaError_t e = run_once_per_device(s_attrs, [] {
    const void* fns[] = {(const void*)tc::kda_tc_chunk_local_kernel<kGateLogCh>,
                         (const void*)tc::kda_tc_chunk_local_kernel<kGateLogTok>,
                         (const void*)tc::kda_tc_chunk_local_kernel<kGateLogitF32>,
                         (const void*)tc::kda_tc_chunk_local_kernel<kGateLogitBf16>};
    for (const void* fn : fns) {
      cudaError_t r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::KA_DYN);
      if (r != cudaSuccess) return r;
    }
    return cudaFuncSetAttribute(tc::kda_tc_state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)tc::KB_DYN);
  });
  if (e != cudaSuccess) return e;
  const int s_sms = current_sm_count();
  if (s_sms <= 0) return cudaErrorInvalidDevice;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int num_seqs = cu_seqlens ? N : 0;
  const long long items = max_chunks * H;
  if (items >= (1LL << 31)) return cudaErrorInvalidValue;  // item indices are 32-bit
  const FastDiv fdH = make_fastdiv((uint32_t)H);
  const FastDiv fdC = make_fastdiv((uint32_t)std::max(1, (T + tc::C - 1) / tc::C));
  // The warp-specialised kernel takes every layout and gate mode;
  // `local_kernel` == 1 keeps every call on the two-CTA kernel.
  const bool use_ws = items > 0 && local_kernel != 1 && (long long)B * T < (1LL << 31) && ws::ws_kernel_available();
  const TcWorkspace lay = tc_workspace_layout(max_chunks, H, N * (long long)H, T, seg_chunks, num_seqs);
  int2* table = reinterpret_cast<int2*>(ws + lay.table);
  int* chunk_total = reinterpret_cast<int*>(table + max_chunks);
  // Precise fallback.  These kernels keep U and E in bf16 and T diag(beta)
  // without its lo part, which is accurate unless some chunk has near-parallel
  // keys (|A_rj| >= kSolveAccurateA: then U's rows telescope and their bf16
  // roundings add up).  The chunk-local kernels raise *esc on such a chunk; the
  // state pass then does nothing and the single-pass kernel, which handles
  // those chunks in its precise form, recomputes the whole call.
  int* esc = reinterpret_cast<int*>(ws + lay.esc);
  if (!fu::fused_kernel_available()) return cudaErrorNotSupported;
  e = fu::launch_fused(q, k, v, g, beta, S0, o, S_out, cu_seqlens, N, B, T, H, ws + lay.fused, s_sms, gmode,
                       stream, fu::kFusedSetup, esc);
  if (e != cudaSuccess) return e;
  if (cu_seqlens) {
    // validates cu_seqlens (a malformed table: total = -1 and every later kernel
    // skips its work) and builds the chunk table of packed sequences
    ws::kda_ws_chunk_table_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, num_seqs, T, table, chunk_total);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (use_ws) {
    e = ws::launch_ws_local(q, k, v, g, beta, cu_seqlens, num_seqs, B, T, H, items, fdH, fdC, ws,
                            reinterpret_cast<uint32_t*>(ws + lay.lists), table, chunk_total, esc,
                            std::min(s_sms, kMaxListCtas), gmode, stream);
    if (e != cudaSuccess) return e;
  } else if (items > 0) {
    const int gridA = (int)(items < 2LL * s_sms ? items : 2LL * s_sms);
#define KDA_TC_LOCAL(M)                                                                            \
  tc::kda_tc_chunk_local_kernel<M><<<gridA, 256, tc::KA_DYN, stream>>>(q, k, v, g, beta, cu_seqlens, \
                                                                       num_seqs, T, H, (uint32_t)items, fdH, \
                                                                       fdC, ws, nullptr, nullptr, 0u, \
                                                                       cu_seqlens ? chunk_total : nullptr, esc)
    switch (gmode) {
      case kGateLogCh: KDA_TC_LOCAL(kGateLogCh); break;
      case kGateLogTok: KDA_TC_LOCAL(kGateLogTok); break;
      case kGateLogitF32: KDA_TC_LOCAL(kGateLogitF32); break;
      case kGateLogitBf16: KDA_TC_LOCAL(kGateLogitBf16); break;
      default: return cudaErrorInvalidValue;
    }
#undef KDA_TC_LOCAL
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (ev && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
  const long long units = (long long)N * H;
  if (units > 0 && seg_chunks > 0 && !cu_seqlens) {
    // segmented: maps of every segment but the last, entry states, final pass
    float* maps = reinterpret_cast<float*>(ws + lay.maps);
    float* seg_init = reinterpret_cast<float*>(ws + lay.seg_init);
    const long long nc = (T + tc::C - 1) / tc::C;
    const int P = (int)((nc + seg_chunks - 1) / seg_chunks);
    const long long map_items = units * (P - 1) * 2, fin_items = units * P;
    tc::kda_tc_state_pass_kernel<<<(int)std::min<long long>(map_items, 2LL * s_sms), 256, tc::KB_DYN, stream>>>(
        ws, S0, S_out, o, nullptr, B, T, H, seg_chunks, tc::kPassMaps, maps, seg_init, nullptr, esc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    tc::kda_tc_seg_combine_kernel<<<(unsigned)(units * (tc::D / 8)), 256, 0, stream>>>(maps, S0, seg_init, P,
                                                                                        esc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    tc::kda_tc_state_pass_kernel<<<(int)std::min<long long>(fin_items, 2LL * s_sms), 256, tc::KB_DYN, stream>>>(
        ws, S0, S_out, o, nullptr, B, T, H, seg_chunks, tc::kPassFinal, maps, seg_init, nullptr, esc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if (units > 0) {
    const int gridB = (int)(units < 2LL * s_sms ? units : 2LL * s_sms);  // two CTAs per SM
    tc::kda_tc_state_pass_kernel<<<gridB, 256, tc::KB_DYN, stream>>>(ws, S0, S_out, o, cu_seqlens, N, T, H, 0,
                                                                      tc::kPassPlain, nullptr, nullptr,
                                                                      cu_seqlens ? chunk_total : nullptr, esc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (units > 0) {
    e = fu::launch_fused(q, k, v, g, beta, S0, o, S_out, cu_seqlens, N, B, T, H, ws + lay.fused, s_sms, gmode,
                         stream, fu::kFusedPrecise, esc);
    if (e != cudaSuccess) return e;
  }
  if (ev && (e = cudaEventRecord(ev[2], stream)) != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace kda
