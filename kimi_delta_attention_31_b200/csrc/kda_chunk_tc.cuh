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
//   E = U - W S,  O = (Q o e^G) S + P E = Q' S + P U  with Q' = Q o e^G - P W,
//   S <- Diag(e^{G_last}) S + (K o e^{G_last - G})^T E.
// Everything left of "S" is chunk-local and parallel over chunks; only the
// last three lines carry the state.  Two kernels:
//
//  1. kda_tc_chunk_local_kernel -- one CTA per (chunk, head), all chunks in
//     parallel.  Builds the decay-scaled bf16 operands in shared memory,
//     computes [A; P] with one tcgen05 MMA (M=128, N=160, K=128) into TMEM,
//     inverts I + A by fp32 forward substitution (warp shuffles), forms
//     W^T, U^T (two MMAs) and (P W)^T (one MMA), and writes a 74,240-byte
//     per-chunk image already laid out as the state pass's MMA operands.
//  2. kda_tc_state_pass_kernel -- persistent, one CTA per SM, one (sequence,
//     head) unit at a time, chunks in order.  The fp32 state lives in
//     registers (thread = state row x 64 columns); per chunk one bulk copy
//     brings the image in (double-buffered) and two MMA groups run:
//       X = [-I; P] U + [W; Q'] S_bf16   -> rows 0..63 = -E, rows 64..127 = O
//       Y = Kbar^T E                     -> S <- gamma o S + Y.
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
#include "kda_common.cuh"
#include "tc_ptx.cuh"

namespace kda {

constexpr bool kTcPathBuilt = true;
constexpr int kTcLaunches = 2;

namespace tc {

using bf16 = __nv_bfloat16;
constexpr int C = 64;   // tokens per chunk
constexpr int D = 128;  // dk = dv

// Per (chunk, head) image: written by the chunk-local kernel, copied in one
// piece by the state pass.  Offsets in bytes; every piece 1024-aligned.
constexpr uint32_t IMG_P = 0;       // P     K-major [64 r][64 j]                 8192
constexpr uint32_t IMG_U = 8192;    // U^T   K-major [128 dv][64 j]               16384
constexpr uint32_t IMG_A1 = 24576;  // [W;Q'] MN-major: 2 panels [128 dk][64 tok] 32768
constexpr uint32_t IMG_KB = 57344;  // Kbar  MN-major: 2 panels [64 tok][64 dk]   16384
constexpr uint32_t IMG_G = 73728;   // gamma = e^{G_last}, fp32 [128]             512
constexpr uint32_t IMG_BYTES = 74240;

// chunk-local kernel shared memory (dynamic, 1024-aligned base)
constexpr uint32_t KA_L3 = 0;       // [K a; Q a]  K-major [128][128] (2 K-panels)  32768
constexpr uint32_t KA_RB = 32768;   // right operands K-major [160][128]          40960
constexpr uint32_t KA_AS = 0;       // after the first MMA: A fp32 [64][65]       16640
constexpr uint32_t KA_PT = 17408;   //                      P bf16 K-major          8192
constexpr uint32_t KA_TT = 25600;   //                      T bf16 K-major          8192
constexpr uint32_t KA_WT = 0;       // after the solve:     W^T bf16 K-major       16384
constexpr uint32_t KA_XK = 73728;   // beta K e^G  MN-major 2 panels [64][64]       16384
constexpr uint32_t KA_BV = 90112;   // beta V      MN-major 2 panels [64][64]       16384
constexpr uint32_t KA_BYTES = 106496;
constexpr uint32_t KA_DYN = KA_BYTES + 1024;

// state-pass kernel shared memory
constexpr uint32_t KB_STAGE = 82944;        // -I (8192) + image (74240) + pad
constexpr uint32_t KB_IMG = 8192;           // image offset inside a stage
constexpr uint32_t KB_SB = 2 * KB_STAGE;    // S bf16 MN-major 2 panels [128][64]  32768
constexpr uint32_t KB_E = KB_SB + 32768;    // E bf16 MN-major 2 panels [64][64]   16384
constexpr uint32_t KB_BYTES = KB_E + 16384;
constexpr uint32_t KB_DYN = KB_BYTES + 1024;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~(uintptr_t)1023);
}
__device__ __forceinline__ void st_bf16(uint8_t* p, float x) {
  *reinterpret_cast<bf16*>(p) = __float2bfloat16_rn(x);
}
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

__device__ __forceinline__ float sel4(int i, float a0, float a1, float a2, float a3) {
  return i == 0 ? a0 : (i == 1 ? a1 : (i == 2 ? a2 : a3));
}

// ---------------------------------------------------------------------------
// Kernel 1: chunk-local work, one CTA (256 threads) per (chunk, head).
// Thread t handles key channel c = t mod 128 for the rows of its half
// (rows 32 * (t / 128) ... + 31) during the gate preparation.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 2)
    kda_tc_chunk_local_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                              const bf16* __restrict__ v, const float* __restrict__ g,
                              const float* __restrict__ beta, const int32_t* __restrict__ cu_seqlens,
                              int num_seqs, int T, int H, uint8_t* __restrict__ ws) {
  __shared__ float s_beta[C];
  __shared__ float s_Ge[4][D];
  __shared__ float s_tot[D];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ uint32_t s_tmem;
  __shared__ long long s_loc_s;
  __shared__ int s_loc_n;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = align1024(dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H;
  const long long ci = blockIdx.x / H;

  long long s0;
  int Cn;
  if (cu_seqlens) {
    if (warp == 0) {
      long long s = 0;
      int cn = 0;
      const bool ok = locate_chunk_warp(cu_seqlens, num_seqs, ci, &s, &cn);
      if (lane == 0) {
        s_loc_s = s;
        s_loc_n = ok ? cn : -1;
      }
    }
    __syncthreads();
    s0 = s_loc_s;
    Cn = s_loc_n;
  } else {
    const long long cps = (T + C - 1) / C;
    const long long cc = ci % cps;
    s0 = (ci / cps) * T + cc * C;
    Cn = (int)min((long long)C, (long long)T - cc * C);
  }
  if (Cn <= 0) return;  // uniform across the CTA

  uint8_t* img = ws + ((size_t)ci * H + h) * IMG_BYTES;
  const int c = tid & 127, half = tid >> 7, r0 = half * 32;
  const uint32_t kp = c >> 6, ce = c & 63;

  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, 256);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&s_bar, 1);
    ptx::fence_mbar_init();
  }
  if (tid < C) s_beta[tid] = tid < Cn ? beta[(size_t)(s0 + tid) * H + h] : 0.f;

  // ---- 1. cumulative log-decay (fp32), rows >= Cn contribute g = 0
  const size_t rs = (size_t)H * D;
  const size_t base = ((size_t)s0 * H + h) * D + c;
  float G[32];
  {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float x = (r0 + i) < Cn ? g[base + (size_t)(r0 + i) * rs] : 0.f;
      acc += x;
      G[i] = acc;
    }
    if (half == 0) s_tot[c] = acc;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (half == 1) {
    const float b0 = s_tot[c];
#pragma unroll
    for (int i = 0; i < 32; ++i) G[i] += b0;
  }
  s_Ge[2 * half][c] = G[15];
  s_Ge[2 * half + 1][c] = G[31];
  __syncthreads();
  const float Ge0 = s_Ge[0][c], Ge1 = s_Ge[1][c], Ge2 = s_Ge[2][c], Ge3 = s_Ge[3][c];

  // ---- 2. decay-scaled bf16 operands
#pragma unroll
  for (int bi = 0; bi < 2; ++bi) {
    const int J = 2 * half + bi;
    const float Gb = J == 0 ? 0.f : sel4(J - 1, Ge0, Ge1, Ge2, Ge3);
    const float GeJ = sel4(J, Ge0, Ge1, Ge2, Ge3);
    const float eGb = expf(Gb);           // e^{G} at the block start
    const float invD = expf(Gb - GeJ);    // 1 / (block decay), >= 1
    const float lam = expf(Ge3 - GeJ);    // decay from block end to chunk end
    // right-operand scale for row block I = J + 1 + t: e^{G_end(I-1) - G_end(J)}
    const float sig1 = J <= 1 ? expf(sel4(J + 1, Ge0, Ge1, Ge2, Ge3) - GeJ) : 0.f;
    const float sig2 = J == 0 ? expf(Ge2 - GeJ) : 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int i = 16 * bi + e;
      const int r = r0 + i;  // == 16 J + e
      float kv = 0.f, qv = 0.f, vv = 0.f;
      if (r < Cn) {
        const size_t off = base + (size_t)r * rs;
        kv = __bfloat162float(k[off]);
        qv = __bfloat162float(q[off]);
        vv = __bfloat162float(v[off]);
      }
      const float a = __expf(G[i] - Gb);
      const float b = __expf(GeJ - G[i]);
      const float br = s_beta[r];
      const float ka = kv * a, kb = kv * b;
      st_bf16(sm + KA_L3 + kp * 16384 + ptx::sw128(r, ce), ka);
      st_bf16(sm + KA_L3 + kp * 16384 + ptx::sw128(64 + r, ce), qv * a);
      // right operands: rows 16 * (I (I - 1) / 2 + J) + e for I = J+1..3, diag at 96 + r
      if (J <= 2) st_bf16(sm + KA_RB + kp * 20480 + ptx::sw128(16 * ((J + 1) * J / 2 + J) + e, ce), kb);
      if (J <= 1) st_bf16(sm + KA_RB + kp * 20480 + ptx::sw128(16 * ((J + 2) * (J + 1) / 2 + J) + e, ce), kb * sig1);
      if (J == 0) st_bf16(sm + KA_RB + kp * 20480 + ptx::sw128(16 * 3 + e, ce), kb * sig2);
      st_bf16(sm + KA_RB + kp * 20480 + ptx::sw128(96 + r, ce), kb * invD);
      // Kbar = K o e^{G_last - G}  (image, MN-major, panel = c / 64, row = token)
      st_bf16(img + IMG_KB + kp * 8192 + ptx::sw128(r, ce), kb * lam);
      // beta K o e^{G} and beta V (MN-major A operands of the WY products)
      st_bf16(sm + KA_XK + kp * 8192 + ptx::sw128(r, ce), br * ka * eGb);
      st_bf16(sm + KA_BV + kp * 8192 + ptx::sw128(r, ce), br * vv);
    }
  }
  if (half == 0) reinterpret_cast<float*>(img + IMG_G)[c] = expf(Ge3);

  // ---- 3. [A'; P'] = [K a; Q a] (right operands)^T : M=128, N=160, K=128
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 160, false, false);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t ad = ptx::sdesc_sw128(sb + KA_L3 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = ptx::sdesc_sw128(sb + KA_RB + (kk >> 2) * 20480 + (kk & 3) * 32, 16, 1024);
      ptx::mma_bf16(tmem, ad, bd, id, kk > 0);
    }
    ptx::mma_commit(&s_bar);
  }
  ptx::mbar_wait_bounded(&s_bar, 0);
  ptx::tc_fence_after();

  // ---- 4. gather A (fp32, beta-scaled, strictly lower) and P (bf16, lower)
  {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int i = tid; i < 1040; i += 256) reinterpret_cast<uint4*>(sm + KA_AS)[i] = z;
    for (int i = tid; i < 512; i += 256) reinterpret_cast<uint4*>(sm + KA_PT)[i] = z;
  }
  __syncthreads();
  {
    const int qd = warp & 3, ch = warp >> 2;
    const int rho = 32 * qd + lane;
    const bool isK = rho < 64;
    const int r = rho & 63, I = r >> 4;
    const float br = s_beta[r];
    float* As = reinterpret_cast<float*>(sm + KA_AS);
#pragma unroll
    for (int grp = 0; grp < 5; ++grp) {
      const int col0 = 80 * ch + 16 * grp;
      float x[16];
      ptx::tmem_ld16(tmem + ((uint32_t)(32 * qd) << 16) + col0, x);
      ptx::tmem_wait_ld();
      int Jb;
      bool use;
      const bool diag = col0 >= 96;
      if (!diag) {
        const int seg = col0 >> 4;
        const int Is = seg == 0 ? 1 : (seg < 3 ? 2 : 3);
        Jb = seg - Is * (Is - 1) / 2;
        use = Is == I;
      } else {
        Jb = (col0 - 96) >> 4;
        use = Jb == I;
      }
      if (use) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = 16 * Jb + e;
          if (isK) {
            if (!diag || j < r) As[r * 65 + j] = br * x[e];
          } else {
            if (!diag || j <= r) st_bf16(sm + KA_PT + ptx::sw128(r, j), x[e]);
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();

  // ---- 5. T = (I + A)^{-1} by forward substitution in fp32.
  // Column j of T is owned by 4 lanes; lane `part` keeps rows i = 4 m + part.
  {
    const float* As = reinterpret_cast<const float*>(sm + KA_AS);
    const int j = tid >> 2, part = tid & 3;
    float x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = (4 * m + part == j) ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 64; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (4 * m < i) acc = fmaf(As[i * 65 + 4 * m + part], x[m], acc);  // A[i][>=i] == 0
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if ((i & 3) == part) x[i >> 2] = (i == j ? 1.f : 0.f) - acc;
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) st_bf16(sm + KA_TT + ptx::sw128(4 * m + part, j), x[m]);
  }

  // ---- 6. W^T = (beta K e^G)^T T^T, U^T = (beta V)^T T^T : M=128, N=64, K=64
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t bd = ptx::sdesc_sw128(sb + KA_TT + kk * 32, 16, 1024);
      ptx::mma_bf16(tmem + 0, ptx::sdesc_sw128(sb + KA_XK + kk * 2048, 8192, 1024), bd, id, kk > 0);
      ptx::mma_bf16(tmem + 64, ptx::sdesc_sw128(sb + KA_BV + kk * 2048, 8192, 1024), bd, id, kk > 0);
    }
    ptx::mma_commit(&s_bar);
  }
  for (int i = tid; i < 512; i += 256)
    reinterpret_cast<uint4*>(img + IMG_P)[i] = reinterpret_cast<const uint4*>(sm + KA_PT)[i];
  ptx::mbar_wait_bounded(&s_bar, 1);
  ptx::tc_fence_after();
  {
    const int qd = warp & 3, ch = warp >> 2;
    const int row = 32 * qd + lane;  // dk channel (W^T) or dv channel (U^T)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float x[32];
      const uint32_t ta = tmem + ((uint32_t)(32 * qd) << 16) + 64 * ch + 32 * hh;
      ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
      ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
      ptx::tmem_wait_ld();
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        const uint4 pk = pack8(x + 8 * k8);
        const uint32_t off = ptx::sw128_chunk(row, 4 * hh + k8);
        if (ch == 0) {
          *reinterpret_cast<uint4*>(img + IMG_A1 + off) = pk;
          *reinterpret_cast<uint4*>(sm + KA_WT + off) = pk;
        } else {
          *reinterpret_cast<uint4*>(img + IMG_U + off) = pk;
        }
      }
    }
  }

  // ---- 7. (P W)^T = W^T P^T : M=128, N=64, K=64; then Q'^T = (Q e^G)^T - (P W)^T
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    ptx::tc_fence_after();
    constexpr uint32_t id = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      ptx::mma_bf16(tmem, ptx::sdesc_sw128(sb + KA_WT + kk * 32, 16, 1024),
                    ptx::sdesc_sw128(sb + KA_PT + kk * 32, 16, 1024), id, kk > 0);
    ptx::mma_commit(&s_bar);
  }
  ptx::mbar_wait_bounded(&s_bar, 0);
  ptx::tc_fence_after();
  {
    const int qd = warp & 3;  // row c = 32 qd + lane == tid mod 128; tokens r0 .. r0 + 31
    float x[32];
    const uint32_t ta = tmem + ((uint32_t)(32 * qd) << 16) + r0;
    ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
    ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
    ptx::tmem_wait_ld();
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = 8 * k8 + e, r = r0 + i;
        const float qv = r < Cn ? __bfloat162float(q[base + (size_t)r * rs]) : 0.f;
        y[e] = qv * __expf(G[i]) - x[i];
      }
      *reinterpret_cast<uint4*>(img + IMG_A1 + 16384 + ptx::sw128_chunk(c, 4 * half + k8)) = pack8(y);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// Kernel 2: the state pass.  Persistent; CTA b handles units b, b + grid, ...
// Thread t: state row c = 32 (warp mod 4) + lane, columns 64 (warp / 4) + [0, 64).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void store_state_bf16(uint8_t* sm, int c, int ch, const float* S) {
#pragma unroll
  for (int k8 = 0; k8 < 8; ++k8)
    *reinterpret_cast<uint4*>(sm + KB_SB + ch * 16384 + ptx::sw128_chunk(c, k8)) = pack8(S + 8 * k8);
}

__global__ void __launch_bounds__(256, 1)
    kda_tc_state_pass_kernel(const uint8_t* __restrict__ ws, const float* __restrict__ S0,
                             float* __restrict__ S_out, bf16* __restrict__ o,
                             const int32_t* __restrict__ cu_seqlens, int N, int T, int H) {
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t s_xbar;
  __shared__ __align__(8) uint64_t s_ybar;
  __shared__ uint32_t s_tmem;
  __shared__ long long s_u_first, s_u_start;
  __shared__ int s_u_len;
  __shared__ int s_abort;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* sm = align1024(dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, ch = warp >> 2;
  const int c = 32 * qd + lane;
  const uint32_t lane_off = (uint32_t)(32 * qd) << 16;

  if (tid == 0) {
    ptx::mbar_init(&s_full[0], 1);
    ptx::mbar_init(&s_full[1], 1);
    ptx::mbar_init(&s_xbar, 1);
    ptx::mbar_init(&s_ybar, 1);
    ptx::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, 256);
    ptx::tmem_relinquish();
  }
  // rows 0..63 of each stage's [-I; P] operand: -I (bf16 -1.0 = 0xBF80)
  for (int idx = tid; idx < 1024; idx += 256) {
    const int stg = idx >> 9, row = (idx >> 3) & 63, chunk = idx & 7;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if ((row >> 3) == chunk) {
      const int e = row & 7;
      w[e >> 1] = (e & 1) ? 0xBF800000u : 0x0000BF80u;
    }
    *reinterpret_cast<uint4*>(sm + stg * KB_STAGE + ptx::sw128_chunk(row, chunk)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tX = s_tmem, tY = s_tmem + 128;

  uint32_t it = 0;          // chunks consumed by this CTA; stage = it & 1
  int pending_stage = -1;   // stage with a copy in flight not yet waited for
  const long long units = (long long)N * H;
  bool aborted = false;
  for (long long u = blockIdx.x; u < units && !aborted; u += gridDim.x) {
    const int n = (int)(u / H), h = (int)(u % H);
    long long first, start;
    int len;
    if (cu_seqlens) {
      if (warp == 0) {
        const long long f = chunks_before_warp(cu_seqlens, n);
        if (lane == 0) {
          s_u_first = f;
          s_u_start = cu_seqlens[n];
          s_u_len = cu_seqlens[n + 1] - cu_seqlens[n];
        }
      }
      __syncthreads();
      first = s_u_first;
      start = s_u_start;
      len = s_u_len;
    } else {
      first = (long long)n * ((T + C - 1) / C);
      start = (long long)n * T;
      len = T;
    }
    const int nc = (len + C - 1) / C;
    const size_t soff = ((size_t)u * D + c) * D + 64 * ch;
    float S[64];
    if (S0) {
#pragma unroll
      for (int j4 = 0; j4 < 16; ++j4) {
        const float4 t = reinterpret_cast<const float4*>(S0 + soff)[j4];
        S[4 * j4] = t.x;
        S[4 * j4 + 1] = t.y;
        S[4 * j4 + 2] = t.z;
        S[4 * j4 + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 64; ++j) S[j] = 0.f;
    }
    store_state_bf16(sm, c, ch, S);
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();

    auto issue = [&](long long chunk_idx, int stage) {
      ptx::mbar_arrive_expect_tx(&s_full[stage], IMG_BYTES);
      ptx::bulk_g2s(sm + stage * KB_STAGE + KB_IMG, ws + ((size_t)chunk_idx * H + h) * IMG_BYTES,
                    IMG_BYTES, &s_full[stage]);
    };
    if (tid == 0 && nc > 0) {
      issue(first, it & 1);
      pending_stage = it & 1;
    }
    for (int cc = 0; cc < nc; ++cc, ++it) {
      const int st = it & 1;
      uint8_t* stage = sm + st * KB_STAGE;
      const uint32_t sst = sb + st * KB_STAGE;
      const long long s = start + (long long)cc * C;
      const int Cn = min(C, len - cc * C);
      if (tid == 0) {
        if (cc + 1 < nc) issue(first + cc + 1, st ^ 1);
        if (!ptx::mbar_wait_bounded(&s_full[st], (it >> 1) & 1)) s_abort = 1;
        pending_stage = (cc + 1 < nc) ? (st ^ 1) : -1;
        ptx::tc_fence_after();
        // X = [-I; P] U  (M=128, N=128, K=64, both K-major)
        constexpr uint32_t id0 = ptx::idesc_bf16(128, 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tX, ptx::sdesc_sw128(sst + kk * 32, 16, 1024),
                        ptx::sdesc_sw128(sst + KB_IMG + IMG_U + kk * 32, 16, 1024), id0, kk > 0);
        // X += [W; Q'] S  (M=128, N=128, K=128, both MN-major)
        constexpr uint32_t id1 = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16(tX, ptx::sdesc_sw128(sst + KB_IMG + IMG_A1 + kk * 2048, 16384, 1024),
                        ptx::sdesc_sw128(sb + KB_SB + kk * 2048, 16384, 1024), id1, 1);
        ptx::mma_commit(&s_xbar);
      }
      if (!ptx::mbar_wait_bounded(&s_xbar, it & 1)) s_abort = 1;
      ptx::tc_fence_after();
      const float gam = reinterpret_cast<const float*>(stage + KB_IMG + IMG_G)[c];
      // epilogue 1: rows 0..63 -> E = -X (bf16 operand), rows 64..127 -> O
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float x[32];
        const uint32_t ta = tX + lane_off + 64 * ch + 32 * hh;
        ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
        ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
        ptx::tmem_wait_ld();
        if (qd < 2) {
#pragma unroll
          for (int k8 = 0; k8 < 4; ++k8) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = -x[8 * k8 + e];
            *reinterpret_cast<uint4*>(sm + KB_E + ch * 8192 + ptx::sw128_chunk(c, 4 * hh + k8)) = pack8(y);
          }
        } else {
          const int r = c - 64;
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
      if (tid == 0) {
        ptx::tc_fence_after();
        // Y = Kbar^T E  (M=128, N=128, K=64, both MN-major)
        constexpr uint32_t id2 = ptx::idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tY, ptx::sdesc_sw128(sst + KB_IMG + IMG_KB + kk * 2048, 8192, 1024),
                        ptx::sdesc_sw128(sb + KB_E + kk * 2048, 8192, 1024), id2, kk > 0);
        ptx::mma_commit(&s_ybar);
      }
      if (!ptx::mbar_wait_bounded(&s_ybar, it & 1)) s_abort = 1;
      ptx::tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float y[32];
        const uint32_t ta = tY + lane_off + 64 * ch + 32 * hh;
        ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(y));
        ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(y + 16));
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) S[32 * hh + e] = fmaf(gam, S[32 * hh + e], y[e]);
      }
      store_state_bf16(sm, c, ch, S);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncthreads();
      if (s_abort) {
        aborted = true;
        break;
      }
    }
    if (!aborted && S_out) {
#pragma unroll
      for (int j4 = 0; j4 < 16; ++j4)
        reinterpret_cast<float4*>(S_out + soff)[j4] =
            make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
    }
  }
  // a copy still in flight after an abort must land before shared memory is released
  if (tid == 0 && aborted && pending_stage >= 0) {
    const uint32_t parity = ((it + 1) >> 1) & 1;
    ptx::mbar_wait_bounded(&s_full[pending_stage], parity);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(s_tmem, 256);
}

}  // namespace tc

inline size_t tc_workspace_bytes(long long max_chunks, int H, int /*N*/) {
  return (size_t)max_chunks * (size_t)H * tc::IMG_BYTES;
}

inline cudaError_t launch_chunk_tc(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                   const __nv_bfloat16* v, const float* g, const float* beta,
                                   const float* S0, __nv_bfloat16* o, float* S_out,
                                   const int32_t* cu_seqlens, int N, int B, int T, int H,
                                   long long max_chunks, void* workspace, cudaEvent_t* ev,
                                   cudaStream_t stream) {
  (void)B;
  static int s_attr_device = -1;
  static int s_sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (s_attr_device != dev) {
    e = cudaFuncSetAttribute(tc::kda_tc_chunk_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::KA_DYN);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc::kda_tc_state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc::KB_DYN);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&s_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    s_attr_device = dev;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int num_seqs = cu_seqlens ? N : 0;
  const long long gridA = max_chunks * H;
  if (gridA > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (gridA > 0) {
    tc::kda_tc_chunk_local_kernel<<<(unsigned)gridA, 256, tc::KA_DYN, stream>>>(
        q, k, v, g, beta, cu_seqlens, num_seqs, T, H, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (ev && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess) return e;
  const long long units = (long long)N * H;
  if (units > 0) {
    const int gridB = (int)(units < s_sms ? units : s_sms);
    tc::kda_tc_state_pass_kernel<<<gridB, 256, tc::KB_DYN, stream>>>(ws, S0, S_out, o, cu_seqlens, N, T,
                                                                      H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (ev && (e = cudaEventRecord(ev[2], stream)) != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace kda
