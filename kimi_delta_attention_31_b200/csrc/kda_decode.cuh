// kda_decode.cuh -- fused recurrent KDA step (decode): one token per
// (sequence, head), state streamed once from HBM and written back in place.
//
// "Deriving Kimi Delta Attention from scratch", section 6 (recurrent mode:
// token-by-token state update for autoregressive decoding); the per-token
// step is that of "Kimi K3 notes 1: KDA", section 5:
//   S~ = Diag(alpha) S,  v^ = S~^T k,  e = beta (v - v^),
//   S <- S~ + k e^T,     o = S^T q = S~^T q + (k . q) e.
// The last rewrite of o is exact algebra; it lets one pass over S~ produce
// both reductions (S~^T k and S~^T q) before anything is written.
//
// Work decomposition: one CTA per (sequence, head, 64-column value block).
// Thread (rg, cq) owns rows rg + 16 i (i < dk/16) of four adjacent value
// columns, loaded as one float4 per row: a warp reads two full 256-byte row
// segments per instruction, so state traffic is perfectly coalesced 128-bit.
// The state never goes through shared memory; only the 2 x dv partial sums
// do.  This is an HBM-streaming kernel: 2 x dk x dv x 4 bytes per head-step.
#pragma once
#include "kda_common.cuh"

namespace kda {

template <typename TIn, int DK, int DV>
struct DecodeCfg {
  static constexpr int DVB = DV < 64 ? DV : 64;  // value columns per CTA
  static constexpr int CQ = DVB / 4;             // float4 column groups
  static constexpr int RG = 16;                  // row groups
  static constexpr int R = DK / RG;              // rows per thread
  static constexpr int NT = CQ * RG;             // threads per CTA
  static constexpr int NWARP = NT / 32;
  static constexpr int NBLK = DV / DVB;          // CTAs per (sequence, head)
  static_assert(DK % RG == 0 && DVB % 4 == 0 && NT % 32 == 0, "shape");
};

template <typename TIn, int DK, int DV, int kGate>
__global__ void __launch_bounds__(DecodeCfg<TIn, DK, DV>::NT)
    kda_decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                           const TIn* __restrict__ v, const void* __restrict__ gate,
                           const float* __restrict__ beta, float* __restrict__ S,
                           TIn* __restrict__ o) {
  constexpr int gmode = kGate;  // GateMode, fixed per instantiation
  using Cfg = DecodeCfg<TIn, DK, DV>;
  constexpr int DVB = Cfg::DVB, CQ = Cfg::CQ, RG = Cfg::RG, R = Cfg::R, NT = Cfg::NT,
                NWARP = Cfg::NWARP;
  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ float s_red[2][NWARP][DVB];
  __shared__ float s_e[DVB];
  __shared__ float s_kq;
  __shared__ float s_nrm[2];

  const int unit = blockIdx.x / Cfg::NBLK;  // n * H + h
  const int vb = blockIdx.x % Cfg::NBLK;
  const int tid = threadIdx.x;
  const int cq = tid % CQ, rg = tid / CQ;
  const int lane = tid & 31, warp = tid >> 5;

  float* Su = S + (size_t)unit * DK * DV + vb * DVB + cq * 4;
  // Issue every state load first: R independent 16-byte loads per thread.
  float4 s[R];
#pragma unroll
  for (int i = 0; i < R; ++i) s[i] = __ldcs(reinterpret_cast<const float4*>(Su + (size_t)(rg + RG * i) * DV));

  for (int c = tid; c < DK; c += NT) {
    s_k[c] = to_f32(k[(size_t)unit * DK + c]);
    s_q[c] = to_f32(q[(size_t)unit * DK + c]);
    s_a[c] = expf(gate_log(gate, gmode, unit, DK, c));
  }
  __syncthreads();
  if constexpr (gate_prep(kGate)) {  // L2-normalise k and q over dk
    if (warp < 2) {
      const float* x = warp == 0 ? s_k : s_q;
      float acc = 0.f;
      for (int c = lane; c < DK; c += 32) acc = fmaf(x[c], x[c], acc);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) s_nrm[warp] = rsqrtf(fmaxf(acc, 1e-24f));
    }
    __syncthreads();
    for (int c = tid; c < DK; c += NT) {
      s_k[c] *= s_nrm[0];
      s_q[c] *= s_nrm[1];
    }
    __syncthreads();
  }
  if (warp == 0) {  // k . q
    float acc = 0.f;
    for (int c = lane; c < DK; c += 32) acc = fmaf(s_k[c], s_q[c], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) s_kq = acc;
  }

  // S~ = Diag(alpha) S and the two reductions S~^T k, S~^T q.
  float4 ak = make_float4(0.f, 0.f, 0.f, 0.f), aq = ak;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int row = rg + RG * i;
    s[i] = f4_scale(s[i], s_a[row]);
    ak = f4_fma(s_k[row], s[i], ak);
    aq = f4_fma(s_q[row], s[i], aq);
  }
#pragma unroll
  for (int off = CQ; off < 32; off <<= 1) {
    ak.x += __shfl_xor_sync(0xffffffffu, ak.x, off);
    ak.y += __shfl_xor_sync(0xffffffffu, ak.y, off);
    ak.z += __shfl_xor_sync(0xffffffffu, ak.z, off);
    ak.w += __shfl_xor_sync(0xffffffffu, ak.w, off);
    aq.x += __shfl_xor_sync(0xffffffffu, aq.x, off);
    aq.y += __shfl_xor_sync(0xffffffffu, aq.y, off);
    aq.z += __shfl_xor_sync(0xffffffffu, aq.z, off);
    aq.w += __shfl_xor_sync(0xffffffffu, aq.w, off);
  }
  if (lane < CQ) {
    *reinterpret_cast<float4*>(&s_red[0][warp][cq * 4]) = ak;
    *reinterpret_cast<float4*>(&s_red[1][warp][cq * 4]) = aq;
  }
  __syncthreads();
  if (tid < DVB) {
    float vhat = 0.f, shat = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) {
      vhat += s_red[0][w][tid];
      shat += s_red[1][w][tid];
    }
    const size_t vi = (size_t)unit * DV + vb * DVB + tid;
    const float e = beta_of(beta, gmode, unit) * (to_f32(v[vi]) - vhat);
    s_e[tid] = e;
    o[vi] = from_f32<TIn>(fmaf(s_kq, e, shat));
  }
  __syncthreads();
  // S <- S~ + k e^T, written back in place.
  const float4 e4 = *reinterpret_cast<const float4*>(&s_e[cq * 4]);
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int row = rg + RG * i;
    const float kr = s_k[row];
    float4 r = s[i];
    r.x = fmaf(kr, e4.x, r.x);
    r.y = fmaf(kr, e4.y, r.y);
    r.z = fmaf(kr, e4.z, r.z);
    r.w = fmaf(kr, e4.w, r.w);
    __stcs(reinterpret_cast<float4*>(Su + (size_t)row * DV), r);
  }
}

template <typename TIn, int DK, int DV>
cudaError_t launch_decode_step(const void* q, const void* k, const void* v, const void* gate,
                               const float* beta, float* S, void* o, int N, int H, int gmode,
                               cudaStream_t stream) {
  using Cfg = DecodeCfg<TIn, DK, DV>;
  const long long grid = (long long)N * H * Cfg::NBLK;
  if (grid == 0) return cudaSuccess;
#define KDA_DECODE_LAUNCH(M)                                                                          \
  kda_decode_step_kernel<TIn, DK, DV, M><<<(unsigned)grid, Cfg::NT, 0, stream>>>(                          \
      static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), gate, beta, S, \
      static_cast<TIn*>(o))
  switch (gmode) {
    case kGateLogCh: KDA_DECODE_LAUNCH(kGateLogCh); break;
    case kGateLogTok: KDA_DECODE_LAUNCH(kGateLogTok); break;
    case kGateLogitF32: KDA_DECODE_LAUNCH(kGateLogitF32); break;
    case kGateLogitBf16: KDA_DECODE_LAUNCH(kGateLogitBf16); break;
    default: return cudaErrorInvalidValue;
  }
#undef KDA_DECODE_LAUNCH
  return cudaGetLastError();
}

}  // namespace kda
