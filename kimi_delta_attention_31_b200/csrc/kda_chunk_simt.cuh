// kda_chunk_simt.cuh -- chunkwise KDA prefill with fp32 arithmetic (CUDA
// cores).  This is the path for fp32 inputs (where bf16/TF32 tensor-core
// operands cannot meet a 1e-4 relative error) and for head sizes or chunk
// sizes the tensor-core path is not built for.
//
// Schedule ("Deriving Kimi Delta Attention from scratch", section 6, chunked
// mode; "Linear / sparse attention" tutorial, section 6.2): for a chunk of C
// tokens entering with state S (dk x dv), G_r = sum_{i<=r} g_i (chunk-relative
// cumulative log-decay, fp32):
//   A_rj = beta_r sum_c k_rc k_jc e^{G_rc-G_jc}        (j <  r)
//   P_rj =        sum_c q_rc k_jc e^{G_rc-G_jc}        (j <= r)
//   (I + A) E = diag(beta) (V - (K o e^G) S)            forward substitution
//   O     = (Q o e^G) S + P E
//   S    <- Diag(e^{G_last}) S + (K o e^{G_last-G})^T E
// Every exponent above is <= 0, so nothing overflows for any gate values.
//
// Work decomposition: one CTA (256 threads) per (sequence, head, 32-column
// value block); value columns of S evolve independently given k, g and beta,
// so the chunk-local A, P are recomputed per value block.  All chunk tiles
// live in shared memory (padded rows: column walks are bank-conflict free).
#pragma once
#include "kda_common.cuh"

namespace kda {

template <int DK, int C>
struct SimtCfg {
  static constexpr int DVB = 32;
  static constexpr int NT = 256;
  static constexpr int LD = DK + 1;   // padded row of a C x dk tile
  static constexpr int LC = C + 1;    // padded row of a C x C tile
  static constexpr int LV = DVB + 1;  // padded row of a C x 32 tile
  static constexpr size_t smem_floats =
      3 * (size_t)C * LD + 2 * (size_t)C * LC + (size_t)DK * DVB + (size_t)C * LV + C + DK;
  static constexpr size_t smem_bytes = smem_floats * sizeof(float);
};

__device__ __forceinline__ void seq_bounds(const int32_t* cu_seqlens, int n, int T, long long* t0,
                                           long long* t1) {
  if (cu_seqlens) {
    checked_seq_range(cu_seqlens, n, T, t0, t1);  // T = total tokens when packed
  } else {
    *t0 = (long long)n * T;
    *t1 = (long long)(n + 1) * T;
  }
}

template <typename TIn, int DK, int C>
__global__ void __launch_bounds__(256)
    kda_chunk_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                          const TIn* __restrict__ v, const void* __restrict__ gate,
                          const float* __restrict__ beta, const float* __restrict__ S0,
                          TIn* __restrict__ o, float* __restrict__ S_out,
                          const int32_t* __restrict__ cu_seqlens, int T, int H, int DV, int gmode) {
  using Cfg = SimtCfg<DK, C>;
  constexpr int DVB = Cfg::DVB, NT = Cfg::NT, LD = Cfg::LD, LC = Cfg::LC, LV = Cfg::LV;
  extern __shared__ float smem[];
  float* Ks = smem;            // k, later K o e^{G_last - G}
  float* Qs = Ks + C * LD;     // q, later Q o e^{G}
  float* Gs = Qs + C * LD;     // G, later K o e^{G}
  float* As = Gs + C * LD;     // beta-scaled strictly lower A
  float* Ps = As + C * LC;     // lower P (with diagonal)
  float* Ss = Ps + C * LC;     // state block [DK][DVB]
  float* Vs = Ss + DK * DVB;   // v block, then right-hand side, then E
  float* bs = Vs + C * LV;     // beta
  float* gl = bs + C;          // G at the last token of the chunk

  const int nvb = DV / DVB;
  const int vb = blockIdx.x % nvb;
  const int uh = blockIdx.x / nvb;  // n * H + h
  const int h = uh % H, n = uh / H;
  const int tid = threadIdx.x;
  long long t0, t1;
  seq_bounds(cu_seqlens, n, T, &t0, &t1);

  // initial state block
  for (int idx = tid; idx < DK * DVB; idx += NT) {
    const int c = idx / DVB, j = idx % DVB;
    Ss[c * DVB + j] = S0 ? S0[((size_t)uh * DK + c) * DV + vb * DVB + j] : 0.f;
  }

  for (long long s = t0; s < t1; s += C) {
    const int Cn = (int)((t1 - s) < C ? (t1 - s) : C);
    __syncthreads();
    // 1. load the chunk (rows >= Cn are zero: g = 0 keeps G flat past the end)
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, c = idx % DK;
      float kv = 0.f, qv = 0.f, gv = 0.f;
      if (r < Cn) {
        const size_t off = ((size_t)(s + r) * H + h) * DK + c;
        kv = to_f32(k[off]);
        qv = to_f32(q[off]);
        gv = gate_log(gate, gmode, (size_t)(s + r) * H + h, DK, c);
      }
      Ks[r * LD + c] = kv;
      Qs[r * LD + c] = qv;
      Gs[r * LD + c] = gv;
    }
    for (int idx = tid; idx < C * DVB; idx += NT) {
      const int r = idx / DVB, j = idx % DVB;
      Vs[r * LV + j] = r < Cn ? to_f32(v[((size_t)(s + r) * H + h) * DV + vb * DVB + j]) : 0.f;
    }
    for (int r = tid; r < C; r += NT) bs[r] = r < Cn ? beta_of(beta, gmode, (size_t)(s + r) * H + h) : 0.f;
    __syncthreads();
    if (gate_prep(gmode)) {  // L2-normalise each row of k and q over dk (a warp per row)
      const int lane = tid & 31;
      for (int r = tid >> 5; r < C; r += NT / 32) {
        float sk = 0.f, sq = 0.f;
        for (int c = lane; c < DK; c += 32) {
          sk = fmaf(Ks[r * LD + c], Ks[r * LD + c], sk);
          sq = fmaf(Qs[r * LD + c], Qs[r * LD + c], sq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sk += __shfl_xor_sync(0xffffffffu, sk, off);
          sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float rk = rsqrtf(fmaxf(sk, 1e-24f)), rq = rsqrtf(fmaxf(sq, 1e-24f));
        for (int c = lane; c < DK; c += 32) {
          Ks[r * LD + c] *= rk;
          Qs[r * LD + c] *= rq;
        }
      }
      __syncthreads();
    }
    // 2. cumulative log-decay per key channel
    for (int c = tid; c < DK; c += NT) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += Gs[r * LD + c];
        Gs[r * LD + c] = acc;
      }
      gl[c] = acc;
    }
    __syncthreads();
    // 3. A and P with pairwise decay ratios (exponent <= 0)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, j = idx % C;
      float a = 0.f, p = 0.f;
      if (j <= r) {
        for (int c = 0; c < DK; ++c) {
          const float w = expf(Gs[r * LD + c] - Gs[j * LD + c]);
          const float kj = Ks[j * LD + c] * w;
          a = fmaf(Ks[r * LD + c], kj, a);
          p = fmaf(Qs[r * LD + c], kj, p);
        }
      }
      As[r * LC + j] = j < r ? bs[r] * a : 0.f;
      Ps[r * LC + j] = p;
    }
    __syncthreads();
    // 4. decay-scaled operands, in place
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, c = idx % DK;
      const float G = Gs[r * LD + c];
      const float eg = expf(G);
      const float kv = Ks[r * LD + c];
      Gs[r * LD + c] = kv * eg;                  // K o e^G
      Qs[r * LD + c] = Qs[r * LD + c] * eg;      // Q o e^G
      Ks[r * LD + c] = kv * expf(gl[c] - G);     // K o e^{G_last - G}
    }
    __syncthreads();
    // 5. right-hand side beta_r (v_r - (k_r o e^{G_r})^T S), in place over V
    for (int idx = tid; idx < C * DVB; idx += NT) {
      const int r = idx / DVB, j = idx % DVB;
      float acc = 0.f;
      for (int c = 0; c < DK; ++c) acc = fmaf(Gs[r * LD + c], Ss[c * DVB + j], acc);
      Vs[r * LV + j] = bs[r] * (Vs[r * LV + j] - acc);
    }
    __syncthreads();
    // 6. forward substitution (I + A) E = rhs: column j owned by 8 lanes of one warp
    {
      const int j = tid >> 3, part = tid & 7;
      for (int r = 1; r < Cn; ++r) {
        float acc = 0.f;
        for (int i = part; i < r; i += 8) acc = fmaf(As[r * LC + i], Vs[i * LV + j], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (part == 0) Vs[r * LV + j] -= acc;
        __syncwarp();
      }
    }
    __syncthreads();
    // 7. outputs O = (Q o e^G) S + P E
    for (int idx = tid; idx < C * DVB; idx += NT) {
      const int r = idx / DVB, j = idx % DVB;
      if (r >= Cn) continue;
      float acc = 0.f;
      for (int c = 0; c < DK; ++c) acc = fmaf(Qs[r * LD + c], Ss[c * DVB + j], acc);
      for (int i = 0; i <= r; ++i) acc = fmaf(Ps[r * LC + i], Vs[i * LV + j], acc);
      o[((size_t)(s + r) * H + h) * DV + vb * DVB + j] = from_f32<TIn>(acc);
    }
    __syncthreads();
    // 8. state hand-off S <- Diag(e^{G_last}) S + (K o e^{G_last-G})^T E
    for (int idx = tid; idx < DK * DVB; idx += NT) {
      const int c = idx / DVB, j = idx % DVB;
      float acc = expf(gl[c]) * Ss[c * DVB + j];
      for (int r = 0; r < Cn; ++r) acc = fmaf(Ks[r * LD + c], Vs[r * LV + j], acc);
      Ss[c * DVB + j] = acc;
    }
  }
  __syncthreads();
  if (S_out) {
    for (int idx = tid; idx < DK * DVB; idx += NT) {
      const int c = idx / DVB, j = idx % DVB;
      S_out[((size_t)uh * DK + c) * DV + vb * DVB + j] = Ss[c * DVB + j];
    }
  }
}

template <typename TIn, int DK, int C>
cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const void* g,
                              const float* beta, const float* S0, void* o, float* S_out,
                              const int32_t* cu_seqlens, int N, int T, int H, int DV, int gmode,
                              cudaStream_t stream) {
  using Cfg = SimtCfg<DK, C>;
  static PerDeviceOnce s_attrs;
  cudaError_t e = run_once_per_device(s_attrs, [] {
    return cudaFuncSetAttribute(kda_chunk_simt_kernel<TIn, DK, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Cfg::smem_bytes);
  });
  if (e != cudaSuccess) return e;
  const long long grid = (long long)N * H * (DV / Cfg::DVB);
  if (grid == 0) return cudaSuccess;
  kda_chunk_simt_kernel<TIn, DK, C><<<(unsigned)grid, Cfg::NT, Cfg::smem_bytes, stream>>>(
      static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), g, beta,
      S0, static_cast<TIn*>(o), S_out, cu_seqlens, T, H, DV, gmode);
  return cudaGetLastError();
}

}  // namespace kda
