// kda_chunk_ws.cuh -- warp-specialised chunk-local kernel for the KDA prefill
// (bf16 q, k, v; dk = dv = 128; C = 64; one sequence per batch row or packed
// sequences; every gate mode: per-channel log-decay, per-token log-decay
// (Gated DeltaNet), or raw per-channel gate logits with the input preparation
// fused).  It computes the same per-(chunk, head) image as
// kda_tc_chunk_local_kernel ("Deriving Kimi Delta Attention from scratch",
// section 6, chunked mode; "Linear / sparse attention" tutorial, section 5.3
// WY representation): P, U^T, [W; Q e^G], Kbar and gamma, on the
// single-reference path.
//
// One CTA per SM, 16 warps in two groups that work on consecutive items at
// the same time:
//   builder (warps 0..7): raw k, q, g rows arrive by tensor-map TMA; the
//     group forms the cumulative log-decays G, the decay-scaled operands
//     K e^G (double-buffered), Q e^G and K e^-G, writes Kbar, Q e^G and
//     gamma to the image, and issues the [A'; P'] MMA into one of two TMEM
//     accumulators.  Its thread 0 starts the next item's TMA as soon as the
//     group has read the raw rows, so that load overlaps the build.
//   solver (warps 8..15): scatters A and P out of TMEM, inverts I + A,
//     issues the W^T / U^T MMAs (V comes straight from TMA in the MMA's
//     layout), and stores P, then U^T and W^T, with bulk copies.  One solver
//     thread outside the solve's serial chains issues its copies and stores.
// Items whose chunk decays below the single-reference range on some channel
// (min G_last < -80) are not built here: the builder appends them to this
// CTA's item list, and the two-CTA kernel runs that list afterwards with the
// 16-token block references.
//
// Hand-offs (all mbarriers, one completion per item unless noted):
//   raw_full      TMA bytes of k, q, g                     builder waits
//   v_full        TMA bytes of V                           solver thread 0 (before the
//                                                          W^T / U^T MMA) or, for a
//                                                          skipped item, the copy thread
//   a_done[slot]  [A'; P'] MMA complete + builder arrive   solver waits; builder
//                 (count 2; per slot: items n, n+2, ...)   waits item n-1's (RB reuse)
//   b_done[slot]  W^T / U^T MMA complete (or skip arrive)  solver waits; builder
//                 (per slot: items n, n+2, ...)            waits item n-2's (slot reuse)
// Per-slot barriers keep every waiter at most one phase behind: the builder
// cannot pass item n+1 before item n-1's b_done, and the solver cannot pass
// item n-1 before item n's a_done, so b_done[slot] is never ahead of item n-2
// when the builder waits for it, and a_done[slot] never ahead of item n when
// the solver does.  Parity waits are therefore exact.
// Every wait is bounded: on a timeout the CTA raises the device error word,
// stops issuing TMA copies and MMAs, runs its remaining items through without
// waiting, and drains what is still in flight before it exits.
//
// Included by kda_chunk_tc.cuh after its kernels (it uses their helpers).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace kda {
namespace ws {

using tc::C;
using tc::D;
using tc::IMG_A1;
using tc::IMG_BYTES;
using tc::IMG_G;
using tc::IMG_KB;
using tc::IMG_P;
using tc::IMG_U;

// shared memory (dynamic, 1024-aligned base)
constexpr uint32_t WS_RAWK = 0;        // k rows [64 tok][128 ch] bf16, row-major             16384
constexpr uint32_t WS_RAWQ = 16384;    // q rows                                               16384
constexpr uint32_t WS_RAWG = 32768;    // g rows [64 tok][128 ch] fp32                         32768
constexpr uint32_t WS_V = 65536;       // V MN-major 2 panels [64 tok][64 dv], 128-B swizzle   16384
// Left operands, K-major, per 64-channel K-panel: K e^G of slot 0 | Q e^G | K e^G of
// slot 1 (64 rows each).  Slot 0's [A'; P'] operand starts at its K rows, slot 1's
// at the Q rows (so its TMEM result has P' in lanes 0..63); the W^T MMA reads K e^G
// of the slot as an MN-major operand.
constexpr uint32_t WS_L3 = 81920;      // 2 panels x 24576                                     49152
constexpr uint32_t WS_L3_PANEL = 24576;
constexpr uint32_t WS_RB = 131072;     // K e^-G K-major 2 panels [64][64]; before the build:
                                       // warp totals of g [8][128] fp32                        16384
constexpr uint32_t WS_UW = 147456;     // staging U^T | W^T (image order)                       32768
constexpr uint32_t WS_AS = 180224;     // A fp32 [64][68], then T over it                      17408
                                       // (free)                                               17408
constexpr uint32_t WS_TT = 215040;     // T diag(beta) bf16 K-major [64][64]; before the solve
                                       // the P staging                                        8192
constexpr uint32_t WS_BYTES = WS_TT + 8192;
constexpr uint32_t WS_DYN = WS_BYTES + 1024;
static_assert(WS_AS + 2 * 17408 == WS_TT && WS_L3 + 2 * WS_L3_PANEL == WS_RB && WS_RB + 16384 == WS_UW &&
                  WS_UW + 32768 == WS_AS, "layout");
static_assert(8 * D * 4 <= 16384, "scratch sizes");
static_assert(WS_TT % 1024 == 0 && WS_RB % 1024 == 0 && WS_L3 % 1024 == 0 && WS_V % 1024 == 0 &&
                  WS_UW % 1024 == 0, "alignment");
static_assert(IMG_A1 - IMG_U == 16384 && IMG_U - IMG_P == 8192, "image order");

// Bytes of one item's raw rows: k, q (bf16) and g -- fp32 per channel, bf16 per
// channel, or none (a per-token gate is read with plain loads: its box would be
// 4 bytes wide, below the 16-byte minimum of a tensor copy).
template <int kGate>
constexpr uint32_t raw_bytes() {
  return 2 * C * D * 2 + (kGate == kGateLogTok ? 0u : kGate == kGateLogitBf16 ? C * D * 2 : C * D * 4);
}
constexpr uint32_t kVBytes = C * D * 2;
constexpr uint32_t kTmemCols = 256;  // [A'; P'] slot 0 | slot 1 | W^T | U^T, 64 columns each
constexpr float kLog2e = 1.4426950408889634f;

struct ItemPos {
  long long s0;  // first token (row of the [tokens, H, D] tensors)
  int h, Cn;     // head, valid rows of the chunk
};
// item = chunk * H + head.  One sequence per batch row: chunk = row * fdC.d +
// chunk-in-row.  Packed sequences: chunk_table[chunk] = {first token, rows}.
template <bool kPacked>
__device__ __forceinline__ ItemPos item_pos(uint32_t item, int T, int H, const FastDiv& fdH, const FastDiv& fdC,
                                            const int2* chunk_table) {
  const uint32_t ci = fdiv(item, fdH);
  ItemPos p;
  p.h = (int)(item - ci * (uint32_t)H);
  if constexpr (kPacked) {
    const int2 e = chunk_table[ci];
    p.s0 = e.x;
    p.Cn = e.y;
  } else {
    const uint32_t bq = fdiv(ci, fdC);
    const int cc = (int)(ci - bq * fdC.d);
    p.s0 = (long long)bq * T + (long long)cc * C;
    p.Cn = min(C, T - cc * C);
  }
  return p;
}

// Chunk table of packed sequences (one CTA of 1024 threads): for every chunk of
// every sequence in order, {first token, rows}; *total = the number of chunks.
// A block-wide exclusive scan of the per-sequence chunk counts, 1024 sequences
// at a time.  First it checks the table it is given: cu_seqlens[0] == 0,
// non-decreasing, cu_seqlens[num_seqs] == T (the total tokens).  A table that
// fails raises the device error word (KDA_ERR_INVALID_ARG) and sets
// *total = -1, which every later kernel of the call reads as "no work"; with a
// valid table the chunk count is at most T / C + num_seqs, the table's capacity.
__global__ void __launch_bounds__(1024)
    kda_ws_chunk_table_kernel(const int32_t* __restrict__ cu_seqlens, int num_seqs, int T,
                              int2* __restrict__ table, int* __restrict__ total) {
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = tid == 0 && (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T);
  for (int i = tid; i < num_seqs; i += 1024) bad |= cu_seqlens[i + 1] < cu_seqlens[i];
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      raise_device_error(kDevErrBadSeqlens);
      *total = -1;
    }
    return;
  }
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < num_seqs; base += 1024) {
    const int i = base + tid;
    int st = 0, len = 0;
    if (i < num_seqs) {
      st = cu_seqlens[i];
      len = cu_seqlens[i + 1] - st;
    }
    const int nch = len > 0 ? (len + C - 1) / C : 0;
    int incl = nch;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += t;
      }
      s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int carry = s_carry;
    const int excl = carry + (warp ? s_warp[warp - 1] : 0) + incl - nch;
    for (int c = 0; c < nch; ++c) table[excl + c] = make_int2(st + c * C, min(C, len - c * C));
    __syncthreads();  // everyone has read s_carry and s_warp
    if (tid == 0) s_carry = carry + s_warp[31];
    __syncthreads();
  }
  if (tid == 0) *total = s_carry;
}

// Bounded wait that also gives up at once when another thread of the CTA has
// already timed out (`abort_flag`), so that a broken hand-off costs one limit,
// not one per remaining item.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              uint64_t limit_ns = 4000000000ull) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      raise_device_error(kDevErrWaitTimeout);
      return false;
    }
  }
}

// kPacked: positions from the chunk table of packed sequences (a template
// parameter, so that the one-row-per-sequence form carries none of it).
template <int kGate, bool kPacked>
__global__ void __launch_bounds__(512, 1)
    kda_ws_chunk_local_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                              const void* __restrict__ gate, const float* __restrict__ beta, int T, int H,
                              uint32_t num_items, FastDiv fdH,
                              FastDiv fdC, uint8_t* __restrict__ ws, uint32_t* __restrict__ steep_list,
                              uint32_t* __restrict__ steep_cnt, uint32_t list_cap,
                              const int2* __restrict__ chunk_table, const int* __restrict__ chunk_total,
                              int* __restrict__ esc_flag) {
  constexpr bool kPrep = gate_prep(kGate);
  constexpr bool kTmaGate = kGate != kGateLogTok;
  __shared__ __align__(16) float s_beta[2][C];
  __shared__ __align__(16) float s_glast[D];  // G at the chunk's last row
  __shared__ float s_nrm[2][C];               // 1 / |k_r|, 1 / |q_r| (only when the call normalises)
  __shared__ __align__(8) uint64_t s_raw_full, s_v_full, s_a_done[2], s_b_done[2], s_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_skip[2];
  __shared__ int s_abort;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  KDA_ALIGNED_DSMEM(sm, dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &s_abort;
  const uint32_t grid = gridDim.x;
  // packed sequences: the exact item count (num_items is the host's upper bound)
  if constexpr (kPacked) num_items = min(num_items, (uint32_t)max(*chunk_total, 0) * (uint32_t)H);

  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tid == 32) {
    ptx::mbar_init(&s_raw_full, 1);
    ptx::mbar_init(&s_v_full, 1);
    ptx::mbar_init(&s_a_done[0], 2);
    ptx::mbar_init(&s_a_done[1], 2);
    ptx::mbar_init(&s_b_done[0], 1);
    ptx::mbar_init(&s_b_done[1], 1);
    ptx::mbar_init(&s_drain, 2);
    s_abort = 0;
    s_skip[0] = s_skip[1] = 0;
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  auto issue_raw = [&](uint32_t item) {
    const ItemPos p = item_pos<kPacked>(item, T, H, fdH, fdC, chunk_table);
    ptx::mbar_arrive_expect_tx(&s_raw_full, raw_bytes<kGate>());
    ptx::tma_load_3d(sm + WS_RAWK, &tm_k, 0, p.h, (int)p.s0, &s_raw_full);
    ptx::tma_load_3d(sm + WS_RAWQ, &tm_q, 0, p.h, (int)p.s0, &s_raw_full);
    if constexpr (kTmaGate) ptx::tma_load_3d(sm + WS_RAWG, &tm_g, 0, p.h, (int)p.s0, &s_raw_full);
  };
  auto issue_v = [&](uint32_t item) {
    const ItemPos p = item_pos<kPacked>(item, T, H, fdH, fdC, chunk_table);
    ptx::mbar_arrive_expect_tx(&s_v_full, kVBytes);
    ptx::tma_load_3d(sm + WS_V, &tm_v, 0, p.h, (int)p.s0, &s_v_full);
    ptx::tma_load_3d(sm + WS_V + 8192, &tm_v, 64, p.h, (int)p.s0, &s_v_full);
  };
  // issued-copy counters of the two issuing threads (for the drain after a timeout)
  uint32_t raw_issued = 0, v_issued = 0;

  if (warp < 8) {
    // ======================= builder =======================
    // thread t owns channels 8 (t mod 16) .. + 7 of rows 4 (t / 16) .. + 3
    const int co = tid & 15, rg = tid >> 4;
    const int c0 = 8 * co;
    const uint32_t kp = co >> 3, ck = co & 7;  // K-panel and 16-byte chunk of the channels
    float* s_wtot = reinterpret_cast<float*>(sm + WS_RB);  // [8 warps][128 ch]
    if (tid == 0) {
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_q);
      if constexpr (kTmaGate) ptx::prefetch_tmap(&tm_g);
      ptx::prefetch_tmap(&tm_v);
      if (blockIdx.x < num_items) {
        issue_raw(blockIdx.x);
        ++raw_issued;
      }
    }
    uint32_t nsteep = 0;
    uint32_t n = 0;
    for (uint32_t item = blockIdx.x; item < num_items; item += grid, ++n) {
      const int slot = n & 1;
      const ItemPos p = item_pos<kPacked>(item, T, H, fdH, fdC, chunk_table);
      float bt = 0.f;
      if (tid < p.Cn) bt = beta_of(beta, kGate, (size_t)(p.s0 + tid) * H + p.h);
      float gtok[4] = {0.f, 0.f, 0.f, 0.f};  // per-token gate of this thread's rows
      if constexpr (kGate == kGateLogTok) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * rg + u < p.Cn) gtok[u] = static_cast<const float*>(gate)[(size_t)(p.s0 + 4 * rg + u) * H + p.h];
      }

      // ---- raw rows to registers; rows >= Cn contribute k = q = 0, g = 0
      wait_or_abort(&s_raw_full, n & 1, abort_flag);
      uint32_t kst[16], qst[16];
      float G[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 4 * rg + u;
        uint4 kw = make_uint4(0, 0, 0, 0), qw = kw;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (r < p.Cn) {
          kw = *reinterpret_cast<const uint4*>(sm + WS_RAWK + r * 256 + 16 * co);
          qw = *reinterpret_cast<const uint4*>(sm + WS_RAWQ + r * 256 + 16 * co);
          if constexpr (kGate == kGateLogTok) {
            a = make_float4(gtok[u], gtok[u], gtok[u], gtok[u]);
            b = a;
          } else if constexpr (kGate == kGateLogitBf16) {
            float x[8];
            tc::unpack8(*reinterpret_cast<const uint4*>(sm + WS_RAWG + r * 256 + 16 * co), x);
            a = make_float4(tc::neg_softplus_sfu(x[0]), tc::neg_softplus_sfu(x[1]), tc::neg_softplus_sfu(x[2]), tc::neg_softplus_sfu(x[3]));
            b = make_float4(tc::neg_softplus_sfu(x[4]), tc::neg_softplus_sfu(x[5]), tc::neg_softplus_sfu(x[6]), tc::neg_softplus_sfu(x[7]));
          } else {
            // the two 16-byte halves in alternating order across the quarter-warp (no bank conflicts)
            const float* gr = reinterpret_cast<const float*>(sm + WS_RAWG + r * 512) + c0;
            const int sw = (co >> 2) & 1;
            const float4 h0 = *reinterpret_cast<const float4*>(gr + 4 * sw);
            const float4 h1 = *reinterpret_cast<const float4*>(gr + 4 - 4 * sw);
            a = sw ? h1 : h0;
            b = sw ? h0 : h1;
            if constexpr (kGate == kGateLogitF32) {
              a = make_float4(tc::neg_softplus_sfu(a.x), tc::neg_softplus_sfu(a.y), tc::neg_softplus_sfu(a.z), tc::neg_softplus_sfu(a.w));
              b = make_float4(tc::neg_softplus_sfu(b.x), tc::neg_softplus_sfu(b.y), tc::neg_softplus_sfu(b.z), tc::neg_softplus_sfu(b.w));
            }
          }
        }
        kst[4 * u] = kw.x; kst[4 * u + 1] = kw.y; kst[4 * u + 2] = kw.z; kst[4 * u + 3] = kw.w;
        qst[4 * u] = qw.x; qst[4 * u + 1] = qw.y; qst[4 * u + 2] = qw.z; qst[4 * u + 3] = qw.w;
        const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) G[u][e] = (u ? G[u - 1][e] : 0.f) + x[e];
      }
      // 1 / |k_r| and 1 / |q_r| over dk (only when the call normalises): the 16
      // lanes of a half-warp hold one row.  Kept in shared memory, not in
      // registers: written before the group's next barrier, read in the build,
      // and not rewritten before the item's last barrier.
      if constexpr (kPrep) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float kx[8], qx[8];
          tc::unpack8(make_uint4(kst[4 * u], kst[4 * u + 1], kst[4 * u + 2], kst[4 * u + 3]), kx);
          tc::unpack8(make_uint4(qst[4 * u], qst[4 * u + 1], qst[4 * u + 2], qst[4 * u + 3]), qx);
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
      // Row-group totals: this warp holds row groups 2w (lanes 0..15) and 2w+1
      // (lanes 16..31) of the same channels; the warp's total goes to s_wtot,
      // which lives in RB: item n-1's [A'; P'] MMA has read RB (and Q e^G) first.
      if (n >= 1) wait_or_abort(&s_a_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag);
      float lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = __shfl_xor_sync(0xffffffffu, G[3][e], 16);
      if (lane >= 16) {
        reinterpret_cast<float4*>(s_wtot + warp * D + c0)[0] =
            make_float4(G[3][0] + lo[0], G[3][1] + lo[1], G[3][2] + lo[2], G[3][3] + lo[3]);
        reinterpret_cast<float4*>(s_wtot + warp * D + c0)[1] =
            make_float4(G[3][4] + lo[4], G[3][5] + lo[5], G[3][6] + lo[6], G[3][7] + lo[7]);
      }
      ptx::bar_sync(1, 256);  // raw rows consumed, warp totals visible
      if (tid == 0 && item + grid < num_items && !*abort_flag) {
        issue_raw(item + grid);
        ++raw_issued;
      }
      {
        float off[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) off[e] = lane >= 16 ? lo[e] : 0.f;
        for (int w2 = 0; w2 < warp; ++w2) {  // warp-uniform
          const float4 t0 = reinterpret_cast<const float4*>(s_wtot + w2 * D + c0)[0];
          const float4 t1 = reinterpret_cast<const float4*>(s_wtot + w2 * D + c0)[1];
          off[0] += t0.x; off[1] += t0.y; off[2] += t0.z; off[3] += t0.w;
          off[4] += t1.x; off[5] += t1.y; off[6] += t1.z; off[7] += t1.w;
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
      // G is non-increasing (g <= 0), so G at the chunk's last row is each channel's minimum
      bool steep = false;
      if (rg == 15) {
        reinterpret_cast<float4*>(s_glast + c0)[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
        reinterpret_cast<float4*>(s_glast + c0)[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
#pragma unroll
        for (int e = 0; e < 8; ++e) steep |= !(G[3][e] >= tc::kChunkRefMinG);
      }
      const bool fast = !ptx::bar_or(1, 256, steep);  // uniform over the group; s_glast visible

      // ---- slot reuse: item n-2's W^T / U^T MMA has read K e^G of this slot (and
      //      the solver is done with TMEM slot, s_beta[slot], s_skip[slot])
      if (n >= 2) wait_or_abort(&s_b_done[slot], ((n - 2) >> 1) & 1, abort_flag);

      if (fast) {
        // Single reference (chunk start): a = e^{G} <= 1, rho = e^{-G} >= 1.
        uint8_t* img = ws + (size_t)item * IMG_BYTES;
        float gl[8], gam[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          gl[e] = s_glast[c0 + e];
          gam[e] = ptx::ex2(gl[e] * kLog2e);
        }
        uint8_t* l3k = sm + WS_L3 + kp * WS_L3_PANEL + (slot ? 16384 : 0);
        uint8_t* l3q = sm + WS_L3 + kp * WS_L3_PANEL + 8192;
        uint8_t* rb = sm + WS_RB + kp * 8192;
        uint32_t qgp[2][8];  // Q e^G of this thread's 4 tokens, bf16 pairs per channel
        float qg_prev[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * rg + u;
          float kv[8], qv[8];
          tc::unpack8(make_uint4(kst[4 * u], kst[4 * u + 1], kst[4 * u + 2], kst[4 * u + 3]), kv);
          tc::unpack8(make_uint4(qst[4 * u], qst[4 * u + 1], qst[4 * u + 2], qst[4 * u + 3]), qv);
          if constexpr (kPrep) tc::normalise_rows(kv, qv, s_nrm[0][r], s_nrm[1][r]);
          float o_ka[8], o_qa[8], o_kr[8], o_kb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float t = G[u][e] * kLog2e;  // G log2(e), in [-115.5, 0]
            const float a = ptx::ex2(t);        // e^G in (0, 1]
            const float rho = ptx::ex2(-t);     // e^-G in [1, e^80]
            o_ka[e] = kv[e] * a;
            o_qa[e] = qv[e] * a;
            o_kr[e] = kv[e] * rho;
            o_kb[e] = o_kr[e] * gam[e];  // K o e^{G_last - G}
            if (u & 1) qgp[u >> 1][e] = ptx::pack_bf16x2(qg_prev[e], o_qa[e]);
            else qg_prev[e] = o_qa[e];
          }
          *reinterpret_cast<uint4*>(l3k + ptx::sw128_chunk(r, ck)) = tc::pack8(o_ka);
          *reinterpret_cast<uint4*>(l3q + ptx::sw128_chunk(r, ck)) = tc::pack8(o_qa);
          *reinterpret_cast<uint4*>(rb + ptx::sw128_chunk(r, ck)) = tc::pack8(o_kr);
          *reinterpret_cast<uint4*>(img + IMG_KB + kp * 8192 + ptx::sw128_chunk(r, ck)) = tc::pack8(o_kb);
        }
        // Q o e^G into the lower panel of the [W; Q e^G] image (MN-major, row = channel,
        // 64 tokens per 128-byte row): this thread's 4 tokens are 8 contiguous bytes
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = c0 + e;
          *reinterpret_cast<uint2*>(img + IMG_A1 + 16384 + c * 128 + ((((4 * rg) >> 3) ^ c) & 7) * 16 +
                                    8 * (rg & 1)) = make_uint2(qgp[0][e], qgp[1][e]);
        }
        if (rg == 0) {
          float gm[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) gm[e] = expf(gl[e]);
          reinterpret_cast<float4*>(img + IMG_G)[2 * co] = make_float4(gm[0], gm[1], gm[2], gm[3]);
          reinterpret_cast<float4*>(img + IMG_G)[2 * co + 1] = make_float4(gm[4], gm[5], gm[6], gm[7]);
        }
      }
      if (tid < C) s_beta[slot][tid] = bt;
      ptx::fence_proxy_async_smem();
      ptx::bar_sync(1, 256);  // operands, s_beta[slot] complete

      if (tid == 0) {
        const bool issue = fast && !*abort_flag;
        if (issue) {
          // ---- [A'; P'] = [K e^G; Q e^G] (K e^-G)^T : M=128, N=64, K=128 (slot 1: [P'; A'])
          ptx::tc_fence_after();
          constexpr uint32_t id = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad =
                ptx::sdesc_sw128(sb + WS_L3 + (kk >> 2) * WS_L3_PANEL + (slot ? 8192 : 0) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = ptx::sdesc_sw128(sb + WS_RB + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
            ptx::mma_bf16(tmem + 64 * slot, ad, bd, id, kk > 0);
          }
          ptx::mma_commit(&s_a_done[slot]);
        }
        if (!fast && nsteep < list_cap) steep_list[(size_t)blockIdx.x * list_cap + nsteep++] = item;
        s_skip[slot] = fast ? 0 : 1;
        ptx::mbar_arrive(&s_a_done[slot]);             // releases s_beta[slot], s_skip[slot]
        if (!issue) ptx::mbar_arrive(&s_a_done[slot]);  // stands in for the MMA completion
      }
    }
    if (tid == 0) steep_cnt[blockIdx.x] = nsteep;
  } else {
    // ======================= solver =======================
    const int st = tid - 256, w8 = warp - 8;
    // Solver thread 0 issues the MMAs; thread kIo (warp 11, which has no part in
    // the solve's serial chains) issues the copies and stores, so that an issue
    // waiting for room in the copy queue never holds up those chains.
    constexpr int kIo = 96;
    if (st == kIo) {
      ptx::prefetch_tmap(&tm_v);
      if (blockIdx.x < num_items) {
        issue_v(blockIdx.x);
        ++v_issued;
      }
    }
    float* As = reinterpret_cast<float*>(sm + WS_AS);
    uint32_t n = 0;
    for (uint32_t item = blockIdx.x; item < num_items; item += grid, ++n) {
      const int slot = n & 1;
      const bool has_next = item + grid < num_items;
      wait_or_abort(&s_a_done[slot], (n >> 1) & 1, abort_flag);
      ptx::tc_fence_after();
      const bool skip = ptx::bar_or(2, 256, s_skip[slot] != 0);
      if (!skip) {
        // ---- scatter A (fp32, beta-scaled) and P (bf16, staged in the T diag(beta) buffer)
        const bool big =
            tc::scatter_single_ref(tmem + 64 * slot, s_beta[slot], As, sm + WS_TT, warp, w8, lane, slot == 1);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        // near-parallel keys: this call's result is recomputed by the single-pass
        // kernel in its precise form (kda_chunk_tc.cuh, launch_chunk_tc)
        if (ptx::bar_or(2, 256, big) && st == 0) *esc_flag = 1;
        if (st == kIo) {
          ptx::bulk_s2g(ws + (size_t)item * IMG_BYTES + IMG_P, sm + WS_TT, 8192);
          ptx::bulk_commit();
        }
        // ---- T = (I + A)^{-1}, T diag(beta) in bf16.  At each barrier thread kIo
        //      first waits for its stores to have read shared memory: T diag(beta)
        //      reuses the P staging (written after the first barrier).
        tc::solve_t_beta<false>(As, s_beta[slot], sm + WS_TT, nullptr, st, w8, lane, [st] {
          if (st == kIo) ptx::bulk_wait_read0();
          ptx::bar_sync(2, 256);
        }, [] {});
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::bar_sync(2, 256);
        // ---- W^T = (K e^G)^T (T diag(beta))^T, U^T = V^T (T diag(beta))^T : M=128, N=64, K=64
        if (st == 0) {
          const bool have_v = wait_or_abort(&s_v_full, n & 1, abort_flag);
          if (have_v && !*abort_flag) {
            ptx::tc_fence_after();
            constexpr uint32_t id = ptx::idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = ptx::sdesc_sw128(sb + WS_TT + kk * 32, 16, 1024);
              const uint64_t xd = ptx::sdesc_sw128(sb + WS_L3 + (slot ? 16384 : 0) + kk * 2048, WS_L3_PANEL, 1024);
              const uint64_t vd = ptx::sdesc_sw128(sb + WS_V + kk * 2048, 8192, 1024);
              ptx::mma_bf16(tmem + 128, xd, bd, id, kk > 0);
              ptx::mma_bf16(tmem + 192, vd, bd, id, kk > 0);
            }
            ptx::mma_commit(&s_b_done[slot]);
          } else {
            ptx::mbar_arrive(&s_b_done[slot]);
          }
        }
        wait_or_abort(&s_b_done[slot], (n >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
        if (st == kIo && has_next && !*abort_flag) {  // V is free again: the next item's V
          issue_v(item + grid);
          ++v_issued;
        }
        tc::stage_w_u(tmem + 128, sm + WS_UW - IMG_U, warp, w8, lane);  // U^T at WS_UW, W^T after it
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::bar_sync(2, 256);
        if (st == kIo) {
          ptx::bulk_s2g(ws + (size_t)item * IMG_BYTES + IMG_U, sm + WS_UW, 32768);
          ptx::bulk_commit();
        }
      } else if (st == kIo) {  // skipped item: keep the V and b_done phases in step
        wait_or_abort(&s_v_full, n & 1, abort_flag);
        ptx::mbar_arrive(&s_b_done[slot]);
        if (has_next && !*abort_flag) {
          issue_v(item + grid);
          ++v_issued;
        }
      }
    }
    if (st == kIo) ptx::bulk_wait0();
  }

  // After a timeout: wait (bounded again) for the copies and MMAs still in
  // flight, so that nothing lands in shared or tensor memory after exit.
  ptx::tc_fence_before();
  __syncthreads();
  if (s_abort) {
    // copies: the builder's thread 0 (raw rows), solver thread 96 (V);
    // MMAs: the builder's thread 0 ([A'; P']) and solver thread 0 (W^T, U^T)
    if (tid == 0 && raw_issued) ptx::mbar_wait_bounded(&s_raw_full, (raw_issued - 1) & 1, 1000000000ull);
    if (tid == 256 + 96 && v_issued) ptx::mbar_wait_bounded(&s_v_full, (v_issued - 1) & 1, 1000000000ull);
    if (tid == 0 || tid == 256) {
      ptx::mma_commit(&s_drain);
      ptx::mbar_wait_bounded(&s_drain, 0, 1000000000ull);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
// cuTensorMapEncodeTiled, fetched once from the driver through the runtime
// (no link against the driver library).
inline cudaError_t tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  static std::mutex mu;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *out = fn;
  return cudaSuccess;
}

// Tensor map over a [tokens, H, 128] tensor (channels contiguous) with a box of
// `box0` channels x 1 head x 64 tokens; rows past the last token read as zero.
inline cudaError_t encode_rows_map(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap* m, const void* base,
                                   bool f32, long long tokens, int H, uint32_t box0, bool swizzle128) {
  const cuuint64_t elt = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)D * elt, (cuuint64_t)H * D * elt};
  const cuuint32_t box[3] = {box0, 1, (cuuint32_t)C};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Whether the warp-specialised kernel fits this device (its shared memory is
// close to the per-block limit); sets the kernel's attribute on first use.
inline bool ws_kernel_available() {
  static PerDeviceOnce once;
  static bool ok[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  run_once_per_device(once, [dev] {
    const void* fns[] = {(const void*)kda_ws_chunk_local_kernel<kGateLogCh, false>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogTok, false>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogitF32, false>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogitBf16, false>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogCh, true>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogTok, true>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogitF32, true>,
                         (const void*)kda_ws_chunk_local_kernel<kGateLogitBf16, true>};
    int optin = 0;
    bool all = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess;
    for (const void* fn : fns) {
      cudaFuncAttributes fa{};
      all = all && cudaFuncGetAttributes(&fa, fn) == cudaSuccess &&
            (size_t)WS_DYN + fa.sharedSizeBytes <= (size_t)optin &&
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WS_DYN) == cudaSuccess;
    }
    ok[dev] = all;
    cudaGetLastError();  // an unavailable kernel is not an error of the call
    return cudaSuccess;
  });
  return ok[dev];
}

// Per-CTA item lists (steep chunks) in the workspace: `grid` lists of `cap`
// entries, then `grid` counts.
inline uint32_t ws_list_cap(long long items, int grid) { return (uint32_t)((items + grid - 1) / grid); }

// Launches the warp-specialised kernel over all items (grid = one CTA per SM)
// and then the two-CTA kernel over the chunks it passed on.
// Packed sequences (cu_seqlens != NULL): first the chunk table, then the
// kernels look positions up in it.
template <int kGate>
inline cudaError_t launch_ws_local_t(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                     const void* g, const float* beta, const int32_t* cu_seqlens, int num_seqs,
                                     int B, int T, int H, long long items, FastDiv fdH, FastDiv fdC, uint8_t* ws,
                                     uint32_t* lists, const int2* table, const int* table_total, int* esc_flag,
                                     int sms, cudaStream_t stream) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = tensor_map_encoder(&enc);
  if (e != cudaSuccess) return e;
  const long long tokens = (long long)B * T;
  CUtensorMap mk, mq, mg, mv;
  if ((e = encode_rows_map(enc, &mk, k, false, tokens, H, D, false)) != cudaSuccess) return e;
  if ((e = encode_rows_map(enc, &mq, q, false, tokens, H, D, false)) != cudaSuccess) return e;
  if ((e = encode_rows_map(enc, &mv, v, false, tokens, H, 64, true)) != cudaSuccess) return e;
  if constexpr (kGate == kGateLogTok) {
    mg = mk;  // not read: a per-token gate takes plain loads
  } else {
    if ((e = encode_rows_map(enc, &mg, g, kGate != kGateLogitBf16, tokens, H, D, false)) != cudaSuccess) return e;
  }
  const int grid = (int)std::min<long long>(items, sms);
  const uint32_t cap = ws_list_cap(items, grid);
  uint32_t* cnt = lists + (size_t)grid * cap;
  if (cu_seqlens)
    kda_ws_chunk_local_kernel<kGate, true><<<grid, 512, WS_DYN, stream>>>(
        mk, mq, mg, mv, g, beta, T, H, (uint32_t)items, fdH, fdC, ws, lists, cnt, cap, table, table_total,
        esc_flag);
  else
    kda_ws_chunk_local_kernel<kGate, false><<<grid, 512, WS_DYN, stream>>>(
        mk, mq, mg, mv, g, beta, T, H, (uint32_t)items, fdH, fdC, ws, lists, cnt, cap, nullptr, nullptr, esc_flag);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  tc::kda_tc_chunk_local_kernel<kGate><<<grid, 256, tc::KA_DYN, stream>>>(
      q, k, v, g, beta, cu_seqlens, cu_seqlens ? num_seqs : 0, T, H, (uint32_t)items, fdH, fdC, ws, lists, cnt, cap,
      cu_seqlens ? table_total : nullptr, esc_flag);
  return cudaGetLastError();
}

inline cudaError_t launch_ws_local(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const void* g, const float* beta, const int32_t* cu_seqlens, int num_seqs, int B,
                                   int T, int H, long long items, FastDiv fdH, FastDiv fdC, uint8_t* ws,
                                   uint32_t* lists, const int2* table, const int* table_total, int* esc_flag,
                                   int sms, int gmode, cudaStream_t stream) {
#define KDA_WS_CASE(M)                                                                                     \
  case M:                                                                                                  \
    return launch_ws_local_t<M>(q, k, v, g, beta, cu_seqlens, num_seqs, B, T, H, items, fdH, fdC, ws, lists, \
                                table, table_total, esc_flag, sms, stream)
  switch (gmode) {
    KDA_WS_CASE(kGateLogCh);
    KDA_WS_CASE(kGateLogTok);
    KDA_WS_CASE(kGateLogitF32);
    KDA_WS_CASE(kGateLogitBf16);
    default:
      return cudaErrorInvalidValue;
  }
#undef KDA_WS_CASE
}

}  // namespace ws
}  // namespace kda
