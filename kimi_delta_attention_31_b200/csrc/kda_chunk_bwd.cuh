// kda_chunk_bwd.cuh -- backward pass of the chunkwise KDA prefill: gradients
// with respect to q, k, v, g = log alpha, beta and the initial state, in fp32
// arithmetic on the CUDA cores.  kGate selects the gate: one per key channel
// (KDA) or one per token and head (Gated DeltaNet, whose dg is the sum over
// channels of the per-channel dg).
//
// The pages give the forward only ("Deriving Kimi Delta Attention from
// scratch", section 6, chunked mode; "Linear / sparse attention" tutorial,
// sections 5.3 and 6.2).  The backward here is the adjoint of that chunk
// algebra, chunk by chunk in reverse with the state gradient carried from
// chunk to chunk.  Per chunk (C tokens entering with state S; G the
// cumulative log-decay, Gam = e^G, L = e^{G_last - G}, Kb = K o L,
// gam = e^{G_last}; M_rj = e^{G_r - G_j} per channel; X_rj = sum_c K_rc K_jc
// M_rjc and A = beta X strictly lower; P_rj = sum_c Q_rc K_jc M_rjc lower with
// the diagonal; T = (I + A)^{-1}; Bk = beta K o Gam, Bv = beta V; W = T Bk,
// U = T Bv, E = U - W S), given dO and dS' (gradient of the chunk's output state):
//   dE  = Kb dS' + P^T dO,   dKb = E dS'^T,   dOS = dO S^T
//   dS  = gam o dS' + (Q o Gam)^T dO - W^T dE          (to the previous chunk)
//   dP  = lower(dO E^T),  dW = -dE S^T,  dT = dE Bv^T + dW Bk^T
//   dBv = T^T dE,  dBk = T^T dW,  dA = -T^T dT T^T (strictly lower), At = beta o dA
//   dV  = beta o dBv;  dbeta = rowsum(dBv o V + dBk o K o Gam + dA o X)
//   dQ  = dOS o Gam + sum_j dP_rj K_j o M_rj
//   dK  = beta dBk o Gam + dKb o L + sum_j At_rj K_j o M_rj
//         + sum_{r >= j} (At_rj K_r + dP_rj Q_r) o M_rj            (as a column)
//   dG  = beta dBk o K o Gam + dOS o Q o Gam - dKb o Kb
//         + sum_j (At_rj K_r K_j + dP_rj Q_r K_j) o M_rj   - (the same summed as a column)
//   dG_last += sum_r dKb o Kb + gam o rowsum(dS' o S);   dg = reverse cumulative sum of dG.
// Every decay factor is e^{x} with x <= 0, so the pass is exact for any gate.
//
// Work decomposition: one CTA of 4 D threads per (sequence, head).  A forward
// sweep stores each chunk's entry state (fp32) in the workspace; the reverse
// sweep reloads it, recomputes the chunk's A, P, T, W, E and applies the
// equations above.  S and dS (D x D fp32) live in shared memory; loops that
// walk them down a column start at a lane-dependent offset so that a warp's
// loads fall in distinct banks.
#pragma once
#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int C = 16;  // tokens per chunk of the backward

template <int D>
struct Cfg {
  static constexpr int NT = 4 * D;  // threads: 4 per key channel
  static constexpr int NTILE = 11;  // C x D tiles
  static constexpr int NSMALL = 9;  // C x C tiles
  static constexpr size_t smem_floats = 2 * (size_t)D * D + (size_t)NTILE * C * D + (size_t)NSMALL * C * C + 2 * C + 2 * D;
  static constexpr size_t smem_bytes = smem_floats * sizeof(float);
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
__device__ __forceinline__ float4 fma4(float a, float4 b, float4 c) {
  return make_float4(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y), fmaf(a, b.z, c.z), fmaf(a, b.w, c.w));
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}
// sum_j X[r][j] Y[c][j] over a row of each (row length D, 16-byte groups
// visited from a lane-dependent start so that a warp's loads of Y rows, which
// differ per lane, fall in distinct banks).
template <int D>
__device__ __forceinline__ float rowdot(const float* xr, const float* yc, int lane) {
  float acc = 0.f;
#pragma unroll 8
  for (int jj = 0; jj < D / 4; ++jj) {
    const int j = 4 * ((jj + lane) & (D / 4 - 1));
    acc = dot4(ld4(xr + j), ld4(yc + j), acc);
  }
  return acc;
}

// Checkpoint slot of chunk `ch` of sequence n: unique over the packed layout.
__device__ __forceinline__ long long ckpt_slot(bool packed, int n, long long t0, int nch_T, int ch) {
  return packed ? (t0 / C + ch + n) : ((long long)n * nch_T + ch);
}

template <typename TIn, int D, int kGate>
__global__ void __launch_bounds__(4 * D)
    kda_chunk_bwd_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                         const float* __restrict__ g, const float* __restrict__ beta,
                         const float* __restrict__ S0, const TIn* __restrict__ dout,
                         const float* __restrict__ dS_T, float* __restrict__ dq, float* __restrict__ dk,
                         float* __restrict__ dv, float* __restrict__ dg, float* __restrict__ dbeta,
                         float* __restrict__ dS0, const int32_t* __restrict__ cu_seqlens, int T, int H,
                         float* __restrict__ ckpt) {
  constexpr int NT = Cfg<D>::NT;
  extern __shared__ float smem[];
  float* Ss = smem;             // S  [D][D]
  float* dSs = Ss + D * D;      // dS [D][D]
  float* Qs = dSs + D * D;      // C x D tiles
  float* Ks = Qs + C * D;
  float* Gs = Ks + C * D;       // cumulative log-decay
  float* GMs = Gs + C * D;      // e^G
  float* ELs = GMs + C * D;     // e^{G_last - G}
  float* dOs = ELs + C * D;
  float* Ws = dOs + C * D;      // W, later dW
  float* Es = Ws + C * D;
  float* dEs = Es + C * D;
  float* R1 = dEs + C * D;      // U, later dOS
  float* R2 = R1 + C * D;       // dKb
  float* Xs = R2 + C * D;       // C x C tiles
  float* As = Xs + C * C;
  float* Ps = As + C * C;
  float* Ts = Ps + C * C;
  float* dPs = Ts + C * C;
  float* dTs = dPs + C * C;
  float* dAs = dTs + C * C;
  float* Mt = dAs + C * C;
  float* Ats = Mt + C * C;      // beta-scaled dA
  float* bs = Ats + C * C;      // beta [C]
  float* dbs = bs + C;          // dbeta accumulation [C]
  float* gam = dbs + C;         // e^{G_last} [D]
  float* dGl = gam + D;         // gam o rowsum(dS' o S) [D]

  const int uh = blockIdx.x;  // n * H + h
  const int h = uh % H, n = uh / H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  static_assert(kGate == kGateLogCh || kGate == kGateLogTok, "log-decay gates only");
  const bool packed = cu_seqlens != nullptr;
  long long t0 = (long long)n * T, t1 = t0 + T;
  if (packed) checked_seq_range(cu_seqlens, n, T, &t0, &t1);  // T = total tokens when packed
  const int nch = (int)((t1 - t0 + C - 1) / C);
  const int nch_T = (T + C - 1) / C;
  auto row_off = [&](long long t) { return ((size_t)t * H + h) * D; };
  auto slot_ptr = [&](int ch) {
    return ckpt + ((size_t)ckpt_slot(packed, n, t0, nch_T, ch) * H + h) * D * D;
  };

  // Chunk `ch` into shared memory (rows >= Cn are zero; g = 0 there keeps G flat).
  auto load_chunk = [&](int ch, bool with_dout) {
    const long long s = t0 + (long long)ch * C;
    const int Cn = min(C, (int)(t1 - s));
    for (int idx = tid; idx < C * D; idx += NT) {
      const int r = idx / D, c = idx % D;
      float qv = 0.f, kv = 0.f, gv = 0.f, ov = 0.f;
      if (r < Cn) {
        const size_t off = row_off(s + r) + c;
        qv = to_f32(q[off]);
        kv = to_f32(k[off]);
        gv = kGate == kGateLogTok ? g[(size_t)(s + r) * H + h] : g[off];
        if (with_dout) ov = to_f32(dout[off]);
      }
      Qs[idx] = qv;
      Ks[idx] = kv;
      Gs[idx] = gv;
      dOs[idx] = ov;
    }
    for (int r = tid; r < C; r += NT) bs[r] = r < Cn ? beta[(size_t)(s + r) * H + h] : 0.f;
    __syncthreads();
    for (int c = tid; c < D; c += NT) {  // cumulative sum per channel
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += Gs[r * D + c];
        Gs[r * D + c] = acc;
      }
      gam[c] = __expf(acc);
    }
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += NT) {
      const int c = idx % D;
      GMs[idx] = __expf(Gs[idx]);
      ELs[idx] = __expf(Gs[(C - 1) * D + c] - Gs[idx]);
    }
    __syncthreads();
    return Cn;
  };

  // X, A, P, T = (I + A)^{-1}, W = T Bk, U = T Bv (into R1), E = U - W S.
  auto chunk_forward = [&](long long s, int Cn, bool with_p) {
    for (int idx = tid; idx < 2 * C * C; idx += NT) {  // two lanes per pair, halves of the channels
      const int pr = idx >> 1, half = idx & 1, r = pr / C, j = pr % C;
      float x = 0.f, p = 0.f;
      if (j <= r) {
        // the pairs of a warp differ in j (rows of K and G): start each at its own channel
        for (int cc = 0; cc < D / 2; ++cc) {
          const int c = half * (D / 2) + ((cc + j) & (D / 2 - 1));
          const float kj = Ks[j * D + c] * __expf(Gs[r * D + c] - Gs[j * D + c]);
          x = fmaf(Ks[r * D + c], kj, x);
          if (with_p) p = fmaf(Qs[r * D + c], kj, p);
        }
      }
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      if (half == 0) {
        Xs[pr] = j < r ? x : 0.f;
        As[pr] = j < r ? bs[r] * x : 0.f;
        Ps[pr] = p;
      }
    }
    __syncthreads();
    if (tid < C) {  // forward substitution, one column per thread
      const int j = tid;
      float col[C];
#pragma unroll
      for (int i = 0; i < C; ++i) {
        float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc = fmaf(-As[i * C + m], col[m], acc);
        col[i] = acc;
      }
#pragma unroll
      for (int i = 0; i < C; ++i) Ts[i * C + j] = col[i];
    }
    __syncthreads();
    for (int idx = tid; idx < C * D; idx += NT) {  // W = T Bk, U = T Bv
      const int r = idx / D, c = idx % D;
      float w = 0.f, u = 0.f;
      for (int m = 0; m <= r; ++m) {
        const float t = Ts[r * C + m] * bs[m];
        w = fmaf(t, Ks[m * D + c] * GMs[m * D + c], w);
        if (m < Cn) u = fmaf(t, to_f32(v[row_off(s + m) + c]), u);
      }
      Ws[idx] = w;
      R1[idx] = u;
    }
    __syncthreads();
    for (int idx = tid; idx < C * D / 4; idx += NT) {  // E = U - W S, four columns per thread
      const int r = idx / (D / 4), j = 4 * (idx % (D / 4));
      float4 acc = ld4(R1 + r * D + j);
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fma4(-Ws[r * D + c], ld4(Ss + c * D + j), acc);
      st4(Es + r * D + j, acc);
    }
    __syncthreads();
  };

  // ---- forward sweep: the entry state of every chunk into the workspace
  for (int idx = tid; idx < D * D; idx += NT) Ss[idx] = S0 ? S0[(size_t)uh * D * D + idx] : 0.f;
  __syncthreads();
  for (int ch = 0; ch < nch; ++ch) {
    float* slot = slot_ptr(ch);
    for (int idx = tid; idx < D * D; idx += NT) slot[idx] = Ss[idx];
    const long long s = t0 + (long long)ch * C;
    const int Cn = load_chunk(ch, false);
    chunk_forward(s, Cn, false);
    for (int idx = tid; idx < D * D / 4; idx += NT) {  // S <- gam o S + Kb^T E
      const int c = idx / (D / 4), j = 4 * (idx % (D / 4));
      float4 acc = ld4(Ss + c * D + j);
      acc = make_float4(gam[c] * acc.x, gam[c] * acc.y, gam[c] * acc.z, gam[c] * acc.w);
#pragma unroll
      for (int r = 0; r < C; ++r) acc = fma4(Ks[r * D + c] * ELs[r * D + c], ld4(Es + r * D + j), acc);
      st4(Ss + c * D + j, acc);
    }
    __syncthreads();
  }

  // ---- reverse sweep
  for (int idx = tid; idx < D * D; idx += NT) dSs[idx] = dS_T ? dS_T[(size_t)uh * D * D + idx] : 0.f;
  __syncthreads();
  for (int ch = nch - 1; ch >= 0; --ch) {
    const float* slot = slot_ptr(ch);
    for (int idx = tid; idx < D * D; idx += NT) Ss[idx] = slot[idx];
    const long long s = t0 + (long long)ch * C;
    const int Cn = load_chunk(ch, true);
    chunk_forward(s, Cn, true);

    // 1. from the old dS': dE = Kb dS' + P^T dO, dKb = E dS'^T (R2), gam o rowsum(dS' o S)
    for (int idx = tid; idx < C * D / 4; idx += NT) {
      const int r = idx / (D / 4), j = 4 * (idx % (D / 4));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fma4(Ks[r * D + c] * ELs[r * D + c], ld4(dSs + c * D + j), acc);
      for (int rr = r; rr < C; ++rr) acc = fma4(Ps[rr * C + r], ld4(dOs + rr * D + j), acc);
      st4(dEs + r * D + j, acc);
    }
    for (int idx = tid; idx < C * D; idx += NT) {
      const int r = idx / D, c = idx % D;
      R2[idx] = rowdot<D>(Es + r * D, dSs + c * D, lane);
    }
    {  // gam o rowsum(dS' o S): four threads per channel, a quarter of the row each
      const int c = tid >> 2, part = tid & 3;
      float acc = 0.f;
      for (int j = part * (D / 4); j < (part + 1) * (D / 4); j += 4) acc = dot4(ld4(dSs + c * D + j), ld4(Ss + c * D + j), acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (part == 0) dGl[c] = gam[c] * acc;
    }
    __syncthreads();
    // 2. dP = lower(dO E^T); dOS = dO S^T (R1, U is no longer needed)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, j = idx % C;
      dPs[idx] = j <= r ? rowdot<D>(dOs + r * D, Es + j * D, lane) : 0.f;
    }
    for (int idx = tid; idx < C * D; idx += NT) {
      const int r = idx / D, c = idx % D;
      R1[idx] = rowdot<D>(dOs + r * D, Ss + c * D, lane);
    }
    __syncthreads();
    // 3. dS = gam o dS' + (Q o Gam)^T dO - W^T dE  (in place: each element reads only itself of dS')
    for (int idx = tid; idx < D * D / 4; idx += NT) {
      const int c = idx / (D / 4), j = 4 * (idx % (D / 4));
      float4 acc = ld4(dSs + c * D + j);
      acc = make_float4(gam[c] * acc.x, gam[c] * acc.y, gam[c] * acc.z, gam[c] * acc.w);
#pragma unroll
      for (int r = 0; r < C; ++r) {
        acc = fma4(Qs[r * D + c] * GMs[r * D + c], ld4(dOs + r * D + j), acc);
        acc = fma4(-Ws[r * D + c], ld4(dEs + r * D + j), acc);
      }
      st4(dSs + c * D + j, acc);
    }
    __syncthreads();
    // 4. dW = -dE S^T (over W)
    for (int idx = tid; idx < C * D; idx += NT) {
      const int r = idx / D, c = idx % D;
      Ws[idx] = -rowdot<D>(dEs + r * D, Ss + c * D, lane);
    }
    for (int idx = tid; idx < C * D; idx += NT) {  // V over E (E is no longer read)
      const int r = idx / D, c = idx % D;
      Es[idx] = r < Cn ? to_f32(v[row_off(s + r) + c]) : 0.f;
    }
    __syncthreads();
    // 5. dT = dE Bv^T + dW Bk^T
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, j = idx % C;
      float acc = 0.f;
      if (j < Cn) {
        for (int dd = 0; dd < D / 4; ++dd) {
          const int d = 4 * ((dd + lane) & (D / 4 - 1));
          acc = dot4(ld4(dEs + r * D + d), ld4(Es + j * D + d), acc);
          const float4 kk = ld4(Ks + j * D + d), gm = ld4(GMs + j * D + d);
          acc = dot4(ld4(Ws + r * D + d), make_float4(kk.x * gm.x, kk.y * gm.y, kk.z * gm.z, kk.w * gm.w), acc);
        }
        acc *= bs[j];
      }
      dTs[idx] = acc;
    }
    __syncthreads();
    // 6. dA = -T^T dT T^T (strictly lower): Mt = dT T^T, then -T^T Mt
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, j = idx % C;
      float acc = 0.f;
      for (int m = 0; m < C; ++m) acc = fmaf(dTs[r * C + m], Ts[j * C + m], acc);
      Mt[idx] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, j = idx % C;
      float acc = 0.f;
      for (int m = 0; m < C; ++m) acc = fmaf(Ts[m * C + r], Mt[m * C + j], acc);
      dAs[idx] = j < r ? -acc : 0.f;
      Ats[idx] = j < r ? -acc * bs[r] : 0.f;
    }
    __syncthreads();
    for (int r = tid; r < C; r += NT) {  // dbeta from A: rowsum(dA o X)
      float acc = 0.f;
      for (int j = 0; j < C; ++j) acc = fmaf(dAs[r * C + j], Xs[r * C + j], acc);
      dbs[r] = acc;
    }
    __syncthreads();
    // 7. per (row, channel) outputs.  Thread (c, part) owns channel c of rows
    //    part, part + 4, ... both as a row (left factor) and as a column (right
    //    factor) of the pairwise terms, so no two threads write one element.
    {
      // a warp covers 32 consecutive channels of one row group: conflict-free tile accesses
      const int c = tid % D, part = tid / D;
      float dQa[C / 4], dKa[C / 4], dGa[C / 4];
      float kbsum = 0.f;  // sum over this thread's rows of dKb o Kb (for G_last)
#pragma unroll
      for (int i = 0; i < C / 4; ++i) {
        const int r = part + 4 * i, e = r * D + c;
        const float Gr = Gs[e], kr = Ks[e], qr = Qs[e];
        // dBv, dBk for this element (T lower: rows m >= r)
        float dbv = 0.f, dbk = 0.f;
        for (int m = r; m < C; ++m) {
          dbv = fmaf(Ts[m * C + r], dEs[m * D + c], dbv);
          dbk = fmaf(Ts[m * C + r], Ws[m * D + c], dbk);
        }
        const float vr = Es[e];
        atomicAdd(&dbs[r], dbv * vr + dbk * kr * GMs[e]);
        if (r < Cn) dv[row_off(s + r) + c] = bs[r] * dbv;
        const float dos = R1[e], dkb = R2[e];
        float dQ = dos * GMs[e];
        float dK = bs[r] * dbk * GMs[e] + dkb * ELs[e];
        float dG = bs[r] * dbk * kr * GMs[e] + dos * qr * GMs[e] - dkb * kr * ELs[e];
        kbsum = fmaf(dkb, kr * ELs[e], kbsum);
        // as a row: pairs (r, j <= r)
        for (int j = 0; j <= r; ++j) {
          const float kj = Ks[j * D + c], w = __expf(Gr - Gs[j * D + c]);
          const float at = Ats[r * C + j], dp = dPs[r * C + j];
          dQ = fmaf(dp * kj, w, dQ);
          dK = fmaf(at * kj, w, dK);
          dG = fmaf((at * kr + dp * qr) * kj, w, dG);
        }
        // as a column: pairs (rr >= r, r)
        for (int rr = r; rr < C; ++rr) {
          const float w = __expf(Gs[rr * D + c] - Gr);
          const float at = Ats[rr * C + r], dp = dPs[rr * C + r];
          const float f = at * Ks[rr * D + c] + dp * Qs[rr * D + c];
          dK = fmaf(f, w, dK);
          dG = fmaf(-f * kr, w, dG);
        }
        dQa[i] = dQ;
        dKa[i] = dK;
        dGa[i] = dG;
      }
      // G_last terms go to the chunk's last row (row C - 1, owned by part 3);
      // the four parts' sums of dKb o Kb meet in shared memory (over Mt/Ats, no longer read)
      float* kbs = Mt;  // [4][D] floats fit in the two C x C tiles Mt, Ats (2 C^2 >= 4 D for D <= 128)
      static_assert(2 * C * C >= 4 * D, "partial sums must fit in Mt and Ats");
      __syncthreads();  // every thread is done reading Ats
      kbs[part * D + c] = kbsum;
      __syncthreads();
      if (part == (C - 1) % 4)
        dGa[C / 4 - 1] += kbs[c] + kbs[D + c] + kbs[2 * D + c] + kbs[3 * D + c] + dGl[c];
      // dQ, dK out; dG into a tile (over dE) for the reverse cumulative sum
#pragma unroll
      for (int i = 0; i < C / 4; ++i) {
        const int r = part + 4 * i;
        if (r < Cn) {
          const size_t o = row_off(s + r) + c;
          dq[o] = dQa[i];
          dk[o] = dKa[i];
        }
      }
      __syncthreads();  // every read of dE is done
#pragma unroll
      for (int i = 0; i < C / 4; ++i) dEs[(part + 4 * i) * D + c] = dGa[i];
      __syncthreads();
      if constexpr (kGate == kGateLogTok) {
        // one gate per token and head (Gated DeltaNet: every key channel decays
        // by the same g_t), so dL/dg_t is the sum over channels of the
        // per-channel gradient: the row sums of dG, then the same reverse
        // cumulative sum (the two sums commute)
        float* rsum = Mt;  // C floats (Mt is no longer read in this chunk)
        for (int r = warp; r < C; r += NT / 32) {
          float acc = 0.f;
          for (int cc = lane; cc < D; cc += 32) acc += dEs[r * D + cc];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) rsum[r] = acc;
        }
        __syncthreads();
        if (tid == 0) {
          float acc = 0.f;
          for (int r = C - 1; r >= 0; --r) {
            acc += rsum[r];
            if (r < Cn) dg[(size_t)(s + r) * H + h] = acc;
          }
        }
      } else if (part == 0) {  // dg_i = sum_{r >= i} dG_r
        float acc = 0.f;
        for (int r = C - 1; r >= 0; --r) {
          acc += dEs[r * D + c];
          if (r < Cn) dg[row_off(s + r) + c] = acc;
        }
      }
    }
    for (int r = tid; r < Cn; r += NT) dbeta[(size_t)(s + r) * H + h] = dbs[r];
    __syncthreads();
  }
  if (dS0)
    for (int idx = tid; idx < D * D; idx += NT) dS0[(size_t)uh * D * D + idx] = dSs[idx];
}

template <typename TIn, int D, int kGate>
cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             const float* S0, const void* dout, const float* dS_T, float* dq, float* dk,
                             float* dv, float* dg, float* dbeta, float* dS0, const int32_t* cu_seqlens, int N,
                             int T, int H, float* ckpt, cudaStream_t stream) {
  static PerDeviceOnce s_attrs;
  cudaError_t e = run_once_per_device(s_attrs, [] {
    return cudaFuncSetAttribute(kda_chunk_bwd_kernel<TIn, D, kGate>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Cfg<D>::smem_bytes);
  });
  if (e != cudaSuccess) return e;
  const long long units = (long long)N * H;
  if (units == 0) return cudaSuccess;
  kda_chunk_bwd_kernel<TIn, D, kGate><<<(unsigned)units, Cfg<D>::NT, Cfg<D>::smem_bytes, stream>>>(
      static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), g, beta, S0,
      static_cast<const TIn*>(dout), dS_T, dq, dk, dv, dg, dbeta, dS0, cu_seqlens, T, H, ckpt);
  return cudaGetLastError();
}

// Workspace (checkpoints): one D x D fp32 state per (chunk of C tokens, head).
inline size_t bwd_workspace_bytes(int B, int T, int H, int D, int num_seqs) {
  const long long slots = num_seqs > 0 ? (long long)T / C + num_seqs : (long long)B * ((T + C - 1) / C);
  return (size_t)slots * H * D * D * sizeof(float);
}

// ---- backward of the prefill from raw projections (kda_chunk_fwd_prep).
// The preparation of that entry point, per token-head row:
//   q^ = q / max(|q|, 1e-12),  k^ likewise,  g = -softplus(a),  beta = sigmoid(b)
// composed with the recurrence, so its gradients are the recurrence's (taken
// on the prepared inputs in fp32) through the preparation's Jacobians:
//   dq = (dq^ - q^ (q^ . dq^)) / |q|   (dq^ / 1e-12 where the clamp holds)
//   da = -sigmoid(a) dg,   db = beta (1 - beta) dbeta.

// Workspace after the checkpoints: fp32 q^, k^ [rows][D], v, dO [rows][D],
// g [rows][D], beta [rows], and the rows' sums of squares of q and k.
struct PrepBwdLayout {
  size_t qn, kn, vf, dof, g, beta, sq, sk, total;
};
inline PrepBwdLayout prep_bwd_layout(size_t ckpt_bytes, long long rows, int D) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  PrepBwdLayout L;
  const size_t mat = up((size_t)rows * D * sizeof(float)), vec = up((size_t)rows * sizeof(float));
  L.qn = up(ckpt_bytes);
  L.kn = L.qn + mat;
  L.vf = L.kn + mat;
  L.dof = L.vf + mat;
  L.g = L.dof + mat;
  L.beta = L.g + mat;
  L.sq = L.beta + vec;
  L.sk = L.sq + vec;
  L.total = L.sk + vec;
  return L;
}

// The preparation, one warp per token-head row, in the forward's arithmetic
// (rsqrt of the clamped sum of squares, the same -softplus and sigmoid).
template <typename TIn, int D>
__global__ void __launch_bounds__(256)
    kda_bwd_prep_in_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                           const TIn* __restrict__ dout, const void* __restrict__ a, int a_bf16,
                           const float* __restrict__ b, float* __restrict__ qn, float* __restrict__ kn,
                           float* __restrict__ vf, float* __restrict__ dof, float* __restrict__ g,
                           float* __restrict__ beta, float* __restrict__ sq, float* __restrict__ sk,
                           long long rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += warps) {
    const size_t base = (size_t)row * D;
    float xq[D / 32], xk[D / 32], ssq = 0.f, ssk = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      xq[i] = to_f32(q[base + lane + 32 * i]);
      xk[i] = to_f32(k[base + lane + 32 * i]);
      ssq = fmaf(xq[i], xq[i], ssq);
      ssk = fmaf(xk[i], xk[i], ssk);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
    }
    const float rq = rsqrtf(fmaxf(ssq, 1e-24f)), rk = rsqrtf(fmaxf(ssk, 1e-24f));
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const size_t e = base + lane + 32 * i;
      qn[e] = xq[i] * rq;
      kn[e] = xk[i] * rk;
      vf[e] = to_f32(v[e]);
      dof[e] = to_f32(dout[e]);
      const float av = a_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a)[e]) : static_cast<const float*>(a)[e];
      g[e] = neg_softplus(av);
    }
    if (lane == 0) {
      beta[row] = sigmoid_f(b[row]);
      sq[row] = ssq;
      sk[row] = ssk;
    }
  }
}

// The chain rule through the preparation, in place over the recurrence's
// gradients: dq, dk (with respect to q^, k^), da (holding dg) and db (holding
// dbeta).  One warp per token-head row.
template <int D>
__global__ void __launch_bounds__(256)
    kda_bwd_prep_out_kernel(const float* __restrict__ qn, const float* __restrict__ kn,
                            const float* __restrict__ sq, const float* __restrict__ sk, const void* __restrict__ a,
                            int a_bf16, const float* __restrict__ beta, float* __restrict__ dq,
                            float* __restrict__ dk, float* __restrict__ da, float* __restrict__ db, long long rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += warps) {
    const size_t base = (size_t)row * D;
    float dqv[D / 32], dkv[D / 32], pq = 0.f, pk = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const size_t e = base + lane + 32 * i;
      dqv[i] = dq[e];
      dkv[i] = dk[e];
      pq = fmaf(qn[e], dqv[i], pq);
      pk = fmaf(kn[e], dkv[i], pk);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pq += __shfl_xor_sync(0xffffffffu, pq, o);
      pk += __shfl_xor_sync(0xffffffffu, pk, o);
    }
    const float ssq = sq[row], ssk = sk[row];
    const float rq = rsqrtf(fmaxf(ssq, 1e-24f)), rk = rsqrtf(fmaxf(ssk, 1e-24f));
    // where the clamp holds, q^ = q / 1e-12 is linear in q: no projection
    if (!(ssq > 1e-24f)) pq = 0.f;
    if (!(ssk > 1e-24f)) pk = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const size_t e = base + lane + 32 * i;
      dq[e] = (dqv[i] - qn[e] * pq) * rq;
      dk[e] = (dkv[i] - kn[e] * pk) * rk;
      const float av = a_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a)[e]) : static_cast<const float*>(a)[e];
      da[e] = -sigmoid_f(av) * da[e];
    }
    if (lane == 0) {
      const float bt = beta[row];
      db[row] = bt * (1.f - bt) * db[row];
    }
  }
}

// The three launches of the raw-projection backward; ws = the workspace
// (checkpoints first, then the layout above).
template <typename TIn, int D>
cudaError_t launch_chunk_bwd_prep(const void* q, const void* k, const void* v, const void* a, int a_bf16,
                                  const float* b, const float* S0, const void* dout, const float* dS_T, float* dq,
                                  float* dk, float* dv, float* da, float* db, float* dS0,
                                  const int32_t* cu_seqlens, int N, int B, int T, int H, size_t ckpt_bytes,
                                  uint8_t* ws, cudaStream_t stream) {
  const long long rows = (long long)B * T * H;
  const PrepBwdLayout L = prep_bwd_layout(ckpt_bytes, rows, D);
  float* qn = reinterpret_cast<float*>(ws + L.qn);
  float* kn = reinterpret_cast<float*>(ws + L.kn);
  float* vf = reinterpret_cast<float*>(ws + L.vf);
  float* dof = reinterpret_cast<float*>(ws + L.dof);
  float* g = reinterpret_cast<float*>(ws + L.g);
  float* beta = reinterpret_cast<float*>(ws + L.beta);
  float* sq = reinterpret_cast<float*>(ws + L.sq);
  float* sk = reinterpret_cast<float*>(ws + L.sk);
  if (rows > 0) {
    const unsigned blocks = (unsigned)std::min<long long>((rows + 7) / 8, 148LL * 16);
    kda_bwd_prep_in_kernel<TIn, D><<<blocks, 256, 0, stream>>>(
        static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v),
        static_cast<const TIn*>(dout), a, a_bf16, b, qn, kn, vf, dof, g, beta, sq, sk, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_chunk_bwd<float, D, kGateLogCh>(qn, kn, vf, g, beta, S0, dof, dS_T, dq, dk, dv, da, db,
                                                         dS0, cu_seqlens, N, T, H,
                                                         reinterpret_cast<float*>(ws), stream);
  if (e != cudaSuccess || rows == 0) return e;
  const unsigned blocks = (unsigned)std::min<long long>((rows + 7) / 8, 148LL * 16);
  kda_bwd_prep_out_kernel<D><<<blocks, 256, 0, stream>>>(qn, kn, sq, sk, a, a_bf16, beta, dq, dk, da, db, rows);
  return cudaGetLastError();
}

}  // namespace bwd
}  // namespace kda
