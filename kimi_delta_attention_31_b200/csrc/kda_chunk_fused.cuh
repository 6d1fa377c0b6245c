// kda_chunk_fused.cuh -- single-pass tensor-core prefill (bf16 q, k, v;
// dk = dv = 128; C = 64): the chunk-local work and the state hand-off of
// every chunk in one persistent kernel, with the carried state kept on chip
// ("Deriving Kimi Delta Attention from scratch", section 6, chunked mode;
// "Linear / sparse attention" tutorial, section 6.2: per chunk an intra term,
// an inter term through the state, and the state handed to the next chunk).
//
// Within a chunk entering with state S (fp32, dk x dv), chunk-relative
// cumulative log-decays G (fp32) and T = (I + A)^{-1} as in kda_chunk_tc.cuh,
// the kernel evaluates
//   W = T diag(beta) (K o e^G),  U = T diag(beta) V,  E = U - W S   (the WY form)
//   O = (Q o e^G) S + P E,       S <- (S + (K o e^-G)^T E) o e^{G_last}
// (the last line is Diag(e^{G_last}) S + (K o e^{G_last - G})^T E with the
// decay applied after the sum; chunks whose decay leaves that range use
// Kbar = K o e^{G_last - G} and decay first).  Nothing of a chunk goes to HBM
// except o, and the final state per (sequence, head) unit.
//
// One CTA per SM (640 threads, ~223 KB of shared memory, all 512 TMEM
// columns).  CTAs take whole units from a counter in the workspace (packed
// sequences longest first) and walk their chunks in order; three warp groups
// work on consecutive chunks at once:
//   builder (warps 0..7)   chunk n+2: cumulative log-decays, the decay-scaled
//                          operands [K e^G; Q e^G] (written over the raw k, q
//                          rows in place) and K e^-G, the [A'; P'] MMA.
//   solver  (warps 8..15)  chunk n+1: A and P out of TMEM and the |A| vote,
//                          T = (I + A)^{-1} and T diag(beta) in bf16, then the
//                          W^T MMA (into the chunk's [A'; P'] columns; read
//                          back and written, negated, in bf16 over the K e^G
//                          rows in their own K-major layout) and the U^T MMA
//                          (straight into the state's columns).
//   state   (warps 16..19) chunk n: the state in TMEM, TRANSPOSED (lane = value
//                          channel), so that every state-side product is an MMA
//                          whose A operand sits in TMEM:
//       [E^T | (Q e^G S)^T] = [U^T | 0] + S^T [-W; Q e^G]^T  (one N=128 group, K=128)
//       S^T  += E^T (K e^-G),  (Q e^G S)^T += E^T P^T          (E as bf16 hi + lo)
//       S^T  *= e^{G_last} per key channel;  o = the second product
// E enters the MMAs as a bf16 pair hi + lo (lo = the rounding error of hi),
// so its fp32 value is used to about 2^-16; U is exact to fp32 accumulation;
// W and S enter in bf16.
//
// Two instances.  The plain one (kPrecise = false) runs every chunk with plain
// TF32 block products and T diag(beta) in bf16.  A chunk whose |A| vote fires
// (some |A_rj| >= kSolveAccurateA: near-parallel keys) needs more: there the
// plain instance marks the unit, and at the unit's end it does not write the
// unit's state (an S_out aliasing S0 keeps S0).  The precise instance, launched
// next, returns at once when no unit is marked and otherwise recomputes the
// marked units, their voted chunks with split-TF32 block products and
// T diag(beta) as a bf16 pair hi + lo (the W and U MMAs run on hi, then lo).
// The precise instance is also the two-kernel path's fallback for the whole
// call (kda_chunk_tc.cuh).
//
// TMEM columns: [A'; P'] slot 0 (0..63) | slot 1 (64..127) (also the W^T
// accumulator) | U^T -> E^T (128..191) | (Q e^G S)^T -> O^T (192..255) | bf16
// hi | lo of E^T (256..319) | S^T bf16 (320..383) | S^T fp32 (384..511).
//
// Copies: builder thread 0 issues the raw gate rows of chunk n+1 once the
// group has read chunk n's; state thread 0 issues k, q of chunk n+2 once chunk
// n's first state MMA has read its panel, and the output tile's two tensor
// stores; solver warp 7, idle in the middle of the solve, issues V of chunk
// n+1 (the slot's V, chunk n-1's, is read by then).  The output tile is staged
// over the chunk's P slot (channels 0..63) and an 8 KB panel (64..127).
//
// Hand-offs (mbarriers; slot = chunk index mod 2):
//   g_full, kq_full[s], v_full[s]   the copies above (bytes)
//   a_done[s]     [A'; P'] MMA complete + builder arrive        -> solver
//   s_ready[s]    solver done (P, -W in shared memory, U^T in TMEM) -> state,
//                 and -> builder (TMEM slot free for chunk n+2)
//   rb_free[s]    state's MMAs of chunk n done (K e^-G read) -> builder
//                 (K e^-G of chunk n+2); gamma has four slots, so the builder
//                 of chunk n+2 never meets chunk n's
//   p_free[s]     chunk n's output tile is read (its P slot and the 8 KB panel
//                 are free) -> solver (P of chunk n+2)
//   x_free        the state has read chunk n's E^T -> the solver's U MMA of
//                 the next chunk may write those columns
//   uw_done, m1, m3, st   MMA completions inside one group.
// Chunk descriptors travel in an 8-entry ring written by builder thread 0
// three chunks ahead.  Every wait is bounded, and every group leaves its loop
// by a group-wide vote, so that after a timeout the whole group stops
// together; the copies still in flight are then waited for (bounded), TMEM is
// freed and the kernel returns with the device error word set.
//
// Included by kda_chunk_tc.cuh after the warp-specialised kernel (it uses
// the tensor-map helpers and the shared solve).
#pragma once

namespace kda {
namespace fu {

using tc::bf16;
using tc::C;
using tc::D;
using ws::wait_or_abort;

// ---------------------------------------------------------- shared memory
constexpr uint32_t FU_L3 = 0;          // 2 slots x 32768: [K e^G; Q e^G] K-major, 2 panels [128 rows][128 B]
constexpr uint32_t FU_L3_SLOT = 32768;
constexpr uint32_t FU_RB = 65536;      // 2 slots x 16384: K e^-G (or Kbar) K-major, 2 panels [64 rows][128 B]
constexpr uint32_t FU_V = 98304;       // 2 slots x 16384: V, two 64-channel panels [64 tokens][128 B]
constexpr uint32_t FU_P = 131072;      // 2 slots x 8192: P bf16 K-major [64 r][64 j]; once read, the
                                       // chunk's output tile, value channels 0..63 ([64 tokens][128 B])
constexpr uint32_t FU_RAWG = 147456;   // raw gate rows [64][128] fp32 (bf16 logits: 16 KB); then the
                                       // group's warp totals [8][128] fp32; steep chunks: left operand
constexpr uint32_t FU_AS = 180224;     // A fp32 [64][68], then T over it
constexpr uint32_t FU_TLO = 197632;    // T diag(beta) bf16, lo part, K-major [64][64]
constexpr uint32_t FU_TT = 205824;     // T diag(beta) bf16, hi part, K-major [64][64]
constexpr uint32_t FU_GAM = 214016;    // 4 slots x 512: gamma = e^{G_last} fp32 [128] (chunk n in slot n mod 4)
constexpr uint32_t FU_OST = 216064;    // the output tile, value channels 64..127 ([64 tokens][128 B])
constexpr uint32_t FU_BYTES = 224256;
constexpr uint32_t FU_DYN = FU_BYTES + 1024;
static_assert(FU_L3 + 2 * FU_L3_SLOT == FU_RB && FU_RB + 2 * 16384 == FU_V && FU_V + 2 * 16384 == FU_P &&
                  FU_P + 2 * 8192 == FU_RAWG && FU_RAWG + 32768 == FU_AS && FU_AS + 17408 == FU_TLO &&
                  FU_TLO + 8192 == FU_TT && FU_TT + 8192 == FU_GAM && FU_GAM + 2048 == FU_OST &&
                  FU_OST + 8192 == FU_BYTES,
              "layout");
static_assert(FU_RB % 1024 == 0 && FU_P % 1024 == 0 && FU_RAWG % 1024 == 0 && FU_TLO % 1024 == 0 &&
                  FU_TT % 1024 == 0 && FU_OST % 1024 == 0, "alignment");
static_assert(8 * D * 4 <= 32768, "scratch sizes");

// ------------------------------------------------------------------ TMEM
constexpr uint32_t kTmCols = 512;
constexpr uint32_t kTmX = 128;   // X^T = S^T [K e^G; Q e^G]^T; E^T (fp32) then lands in its first 64 columns
constexpr uint32_t kTmO = 192;   // (Q e^G S)^T, then O^T
constexpr uint32_t kTmHL = 256;  // bf16 hi (256..287) and lo (288..319) of R^T, then of E^T
constexpr uint32_t kTmSb = 320;  // S^T bf16
constexpr uint32_t kTmS = 384;   // S^T fp32

constexpr int kThreads = 640;  // builder 256, solver 256, state 128
constexpr float kLog2e = 1.4426950408889634f;

// Chunk descriptor.
enum : int { kItFirst = 1, kItLast = 2, kItEmpty = 4, kItEnd = 8, kItSteep = 16 };
struct FuItem {
  long long s0;  // first token (row of the [tokens, H, D] tensors)
  int unit;      // sequence * H + head
  int Cn;        // valid rows (0 for an empty sequence)
  int flags;
  int ord;       // the unit's ordinal among this CTA's units
};

template <int kGate>
constexpr uint32_t g_bytes() {
  return kGate == kGateLogTok ? 0u : kGate == kGateLogitBf16 ? C * D * 2 : C * D * 4;
}
constexpr uint32_t kKqBytes = 4 * 8192, kVBytes = 16384;

// The two bf16 of a 32-bit word as floats (element 2i in the low half).
__device__ __forceinline__ float2 bf2(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}
__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// A block of 32 channels x 32 tokens of a transposed tile in TMEM (lane =
// channel, column = token; `ta` = the warp's first lane and the block's first
// column), times `sign`, as bf16 into a K-major tile in shared memory at
// `tile`: row = token, 128-byte rows of 64 channels with the 128-byte swizzle,
// channels 64..127 `panel` bytes further.  c0 and t0 are the block's first
// channel and token in the tile.  8 x 8 pieces go through stmatrix with
// transposition, so that each token's 8 channels are one 16-byte store.  One
// warp; the roundings are those of a per-element bf16 conversion.
__device__ __forceinline__ void store_tile_t(uint32_t ta, uint32_t tile, int c0, int t0, uint32_t panel, float sign,
                                             int lane) {
  const int piece = lane >> 3, row = lane & 7;  // the row of stmatrix piece `piece` this thread addresses
#pragma unroll
  for (int hl = 0; hl < 2; ++hl) {  // channels c0 + 16 hl .. + 15
    float x[16];
    ptx::tmem_ld16x256b_x4(ta + ((uint32_t)(16 * hl) << 16), x);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {  // tokens t0 + 16 hf .. + 15: pieces (8 tokens) x (channels +0, +8)
      const int c = c0 + 16 * hl + 8 * (piece & 1);
      const int t = t0 + 16 * hf + 8 * (piece >> 1) + row;
      const uint32_t addr = tile + (uint32_t)(c >> 6) * panel + t * 128 + (((((c & 63) >> 3) ^ t) & 7) << 4);
      const float* y = x + 8 * hf;
      ptx::stmatrix_x4_trans(addr, ptx::pack_bf16x2(sign * y[0], sign * y[1]),
                             ptx::pack_bf16x2(sign * y[2], sign * y[3]), ptx::pack_bf16x2(sign * y[4], sign * y[5]),
                             ptx::pack_bf16x2(sign * y[6], sign * y[7]));
    }
  }
}

// One 32-column TMEM load into registers (two 16-column loads).
__device__ __forceinline__ void ld32(uint32_t ta, float* x) {
  ptx::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(x));
  ptx::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(x + 16));
}

// Splits x[0..31] (fp32, tokens 32h .. 32h + 31) into bf16 hi + lo pairs and
// stores them, two tokens per column (token 2i in the low half), at columns
// [base + 16h, +16) (hi) and [base + 32 + 16h, +16) (lo): after both halves
// the 64 tokens' hi parts fill [base, base + 32) and the lo parts the next 32.
__device__ __forceinline__ void store_hi_lo32(uint32_t base, int h, const float* x) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = x[2 * i], b = x[2 * i + 1];
    const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    const float2 f = __bfloat1622float2(p);
    hi[i] = *reinterpret_cast<const uint32_t*>(&p);
    lo[i] = ptx::pack_bf16x2(a - f.x, b - f.y);
  }
  ptx::tmem_st16u(base + 16 * h, hi);
  ptx::tmem_st16u(base + 32 + 16 * h, lo);
}

// Zeroes 64 fp32 TMEM columns [ta, ta + 64) of the calling warp's 32 lanes.
__device__ __forceinline__ void zero_cols64(uint32_t ta) {
  float z[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) z[i] = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) ptx::tmem_st16(ta + 16 * i, z);
}

template <int kGate, bool kPacked, bool kPrecise>
__global__ void __launch_bounds__(kThreads, 1)
    kda_fused_prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                             const __grid_constant__ CUtensorMap tm_o,
                             const void* __restrict__ gate, const float* __restrict__ beta,
                             const float* __restrict__ S0, bf16* __restrict__ o, float* __restrict__ S_out,
                             const int32_t* __restrict__ cu_seqlens, int N, int T, int H,
                             int* __restrict__ unit_ctr, const int* __restrict__ seq_order,
                             const int* __restrict__ seq_status, const int* __restrict__ esc_flag,
                             int* __restrict__ unit_mark, int* __restrict__ any_mark) {
  constexpr bool kPrep = gate_prep(kGate);
  constexpr bool kTmaGate = kGate != kGateLogTok;
  __shared__ __align__(16) float s_beta[2][C];
  __shared__ __align__(16) float s_glast[D];     // G at the chunk's last row
  __shared__ __align__(16) float s_gref[4][D];   // G at the end of each 16-token block (steep chunks)
  __shared__ float s_nrm[2][C];                  // 1 / |k_r|, 1 / |q_r| (only when the call normalises)
  __shared__ FuItem s_ring[8];
  __shared__ __align__(8) uint64_t s_g_full, s_kq_full[2], s_v_full[2], s_a_done[2], s_s_ready[2], s_rb_free[2];
  __shared__ __align__(8) uint64_t s_x_free, s_uw_done, s_m1, s_m3, s_st, s_drain, s_p_free[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_doom[4];  // plain instance: unit (ordinal mod 4) met a chunk with near-parallel keys
  __shared__ int s_kq_mode;  // the state's k, q copies of the coming chunk: 1 = the four copies are armed
  // packed sequences whose cu_seqlens the set-up kernel rejected: no work at all
  if (kPacked && *seq_status < 0) return;
  // the precise instance, run after the plain one (or after the two-kernel
  // path): nothing to do unless a chunk with near-parallel keys was met
  if (esc_flag && *esc_flag == 0) return;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  KDA_ALIGNED_DSMEM(sm, dsm_raw);
  const uint32_t sb = ptx::smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &s_abort;
  const int units = N * H;

  // chunk generator (builder thread 0 only): whole units from the counter.
  // Its state lives in shared memory, so that it holds no registers in the
  // other threads of the group.
  __shared__ struct {
    long long t0;
    int c, nc, len, unit, done, ord;
  } s_gen;
  int& g_c = s_gen.c;
  int& g_nc = s_gen.nc;
  int& g_len = s_gen.len;
  int& g_unit = s_gen.unit;
  int& g_done = s_gen.done;
  long long& g_t0 = s_gen.t0;
  auto gen = [&](FuItem& it) {
    if (g_done) {
      it.flags = kItEnd;
      return;
    }
    if (g_c >= g_nc) {
      int seq;
      for (;;) {
        const int u = atomicAdd(unit_ctr, 1);
        if (u >= units) {
          g_done = 1;
          it.flags = kItEnd;
          return;
        }
        const int rank = u / H, hh = u - rank * H;
        seq = seq_order ? seq_order[rank] : rank;
        g_unit = seq * H + hh;
        // the precise instance after the plain one takes only the units it marked
        if (!kPrecise || !unit_mark || unit_mark[g_unit]) break;
      }
      ++s_gen.ord;
      if constexpr (kPacked) {
        long long a, b;
        checked_seq_range(cu_seqlens, seq, T, &a, &b);
        g_t0 = a;
        g_len = (int)(b - a);
      } else {
        g_t0 = (long long)seq * T;
        g_len = T;
      }
      g_nc = (g_len + C - 1) / C;
      g_c = 0;
      if (g_nc == 0) {  // an empty sequence: one descriptor, S_out = S0
        it.s0 = g_t0;
        it.unit = g_unit;
        it.Cn = 0;
        it.flags = kItFirst | kItLast | kItEmpty;
        it.ord = s_gen.ord;
        return;
      }
    }
    it.s0 = g_t0 + (long long)g_c * C;
    it.unit = g_unit;
    it.ord = s_gen.ord;
    it.Cn = min(C, g_len - g_c * C);
    it.flags = (g_c == 0 ? kItFirst : 0) | (g_c == g_nc - 1 ? kItLast : 0);
    ++g_c;
  };

  if (warp == 0) {
    ptx::tmem_alloc(&s_tmem, kTmCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&s_g_full, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s_kq_full[i], 1);
      ptx::mbar_init(&s_v_full[i], 1);
      ptx::mbar_init(&s_a_done[i], 2);
      ptx::mbar_init(&s_s_ready[i], 1);
      ptx::mbar_init(&s_rb_free[i], 1);
      ptx::mbar_init(&s_p_free[i], 1);
    }
    ptx::mbar_init(&s_x_free, 1);
    ptx::mbar_init(&s_uw_done, 1);
    ptx::mbar_init(&s_m1, 1);
    ptx::mbar_init(&s_m3, 1);
    ptx::mbar_init(&s_st, 1);
    ptx::mbar_init(&s_drain, 3);
    s_abort = 0;
    ptx::fence_mbar_init();
    g_c = g_nc = g_len = g_unit = g_done = 0;
    s_gen.ord = 0;
    for (int i = 0; i < 4; ++i) s_doom[i] = 0;
    g_t0 = 0;
    for (int i = 0; i < 3; ++i) gen(s_ring[i]);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  // TMA of chunk item n's k, q (two 64-channel boxes each, swizzled into the
  // operand panels of slot n & 1), and of its V (slot n & 1); an empty chunk
  // completes the phase with a plain arrive, the end of the work issues nothing.
  auto issue_kq = [&](uint32_t n, uint32_t* issued) {
    const FuItem it = s_ring[n & 7];
    if (it.flags & kItEnd) return;
    const int s = n & 1;
    ++issued[s];
    if ((it.flags & kItEmpty) || *abort_flag) {
      ptx::mbar_arrive(&s_kq_full[s]);
      return;
    }
    const int h = it.unit % H;
    uint8_t* l3 = sm + FU_L3 + s * FU_L3_SLOT;
    ptx::mbar_arrive_expect_tx(&s_kq_full[s], kKqBytes);
    ptx::tma_load_3d(l3, &tm_k, 0, h, (int)it.s0, &s_kq_full[s]);
    ptx::tma_load_3d(l3 + 16384, &tm_k, 64, h, (int)it.s0, &s_kq_full[s]);
    ptx::tma_load_3d(l3 + 8192, &tm_q, 0, h, (int)it.s0, &s_kq_full[s]);
    ptx::tma_load_3d(l3 + 16384 + 8192, &tm_q, 64, h, (int)it.s0, &s_kq_full[s]);
  };
  // The same copies in two steps: arm_kq (one thread) arms the barrier, or
  // completes the phase with a plain arrive when there is nothing to copy, and
  // returns 1 when the four copies are to follow; issue_kq_part(n, p) issues
  // copy p (k or q, channels 0..63 or 64..127).
  auto arm_kq = [&](uint32_t n, uint32_t* issued) -> int {
    const FuItem it = s_ring[n & 7];
    if (it.flags & kItEnd) return 0;
    const int s = n & 1;
    ++issued[s];
    if ((it.flags & kItEmpty) || *abort_flag) {
      ptx::mbar_arrive(&s_kq_full[s]);
      return 0;
    }
    ptx::mbar_arrive_expect_tx(&s_kq_full[s], kKqBytes);
    return 1;
  };
  auto issue_kq_part = [&](uint32_t n, int p) {
    const FuItem it = s_ring[n & 7];
    const int s = n & 1;
    uint8_t* l3 = sm + FU_L3 + s * FU_L3_SLOT;
    ptx::tma_load_3d(l3 + (p & 1) * 16384 + (p >> 1) * 8192, (p >> 1) ? &tm_q : &tm_k, 64 * (p & 1), it.unit % H,
                     (int)it.s0, &s_kq_full[s]);
  };
  auto issue_v = [&](uint32_t n, uint32_t* issued) {
    const FuItem it = s_ring[n & 7];
    if (it.flags & kItEnd) return;
    const int s = n & 1;
    ++issued[s];
    if ((it.flags & kItEmpty) || *abort_flag) {
      ptx::mbar_arrive(&s_v_full[s]);
      return;
    }
    ptx::mbar_arrive_expect_tx(&s_v_full[s], kVBytes);
    ptx::tma_load_3d(sm + FU_V + s * 16384, &tm_v, 0, it.unit % H, (int)it.s0, &s_v_full[s]);
    ptx::tma_load_3d(sm + FU_V + s * 16384 + 8192, &tm_v, 64, it.unit % H, (int)it.s0, &s_v_full[s]);
  };
  // TMA of item n's raw gate rows (per-channel gates only).
  auto issue_g = [&](uint32_t n, uint32_t* issued) {
    if constexpr (kTmaGate) {
      const FuItem it = s_ring[n & 7];
      if (it.flags & kItEnd) return;
      ++*issued;
      if ((it.flags & kItEmpty) || *abort_flag) {
        ptx::mbar_arrive(&s_g_full);
        return;
      }
      ptx::mbar_arrive_expect_tx(&s_g_full, g_bytes<kGate>());
      ptx::tma_load_3d(sm + FU_RAWG, &tm_g, 0, it.unit % H, (int)it.s0, &s_g_full);
    }
  };
  bool mma_issued = false;  // by this thread (builder, solver, state thread 0)
  // copies issued per barrier phase stream (builder thread 0: g; state thread 0: k, q;
  // solver thread 224: V)
  uint32_t g_issued = 0, kq_issued[2] = {0u, 0u}, v_issued[2] = {0u, 0u};

  if (warp < 8) {
    // ============================== builder ==============================
    // thread t owns channels 8 (t mod 16) .. + 7 of rows 4 (t / 16) .. + 3
    const int co = tid & 15, rg = tid >> 4;
    const int c0 = 8 * co;
    const uint32_t kp = co >> 3, ck = co & 7;  // 64-channel panel and 16-byte chunk of the channels
    float* s_wtot = reinterpret_cast<float*>(sm + FU_RAWG);  // [8 warps][128 ch]
    if (tid == 0) {
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_q);
      if constexpr (kTmaGate) ptx::prefetch_tmap(&tm_g);
      ptx::prefetch_tmap(&tm_v);
      ptx::prefetch_tmap(&tm_o);
      issue_g(0, &g_issued);
    }
    uint32_t st_round = 0;  // completions of s_st
    for (uint32_t n = 0;; ++n) {
      const int s = n & 1;
      if (tid == 0) gen(s_ring[(n + 3) & 7]);
      const FuItem it = s_ring[n & 7];
      if (it.flags & kItEnd) {
        if (tid == 0) {
          ptx::mbar_arrive(&s_a_done[s]);
          ptx::mbar_arrive(&s_a_done[s]);
        }
        break;
      }
      if (it.flags & kItEmpty) {  // keep the per-chunk phases in step; nothing to build
        bool okE = true;
        if constexpr (kTmaGate) okE = wait_or_abort(&s_g_full, n & 1, abort_flag);
        if (ptx::bar_or(1, 256, !okE || *abort_flag)) break;  // uniform over the group
        if (tid == 0) {
          issue_g(n + 1, &g_issued);
          ptx::mbar_arrive(&s_a_done[s]);
          ptx::mbar_arrive(&s_a_done[s]);
        }
        continue;
      }
      const int h = it.unit % H;
      const long long s0 = it.s0;
      const int Cn = it.Cn;
      uint8_t* l3 = sm + FU_L3 + s * FU_L3_SLOT;
      uint8_t* rb = sm + FU_RB + s * 16384;
      float bt = 0.f;
      if (tid < Cn) bt = beta_of(beta, kGate, (size_t)(s0 + tid) * H + h);
      float gtok[4] = {0.f, 0.f, 0.f, 0.f};  // per-token gate of this thread's rows
      if constexpr (kGate == kGateLogTok) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (4 * rg + u < Cn) gtok[u] = static_cast<const float*>(gate)[(size_t)(s0 + 4 * rg + u) * H + h];
      }
      // Every wait is followed by a group-wide vote before anything depends on
      // it, so that the whole group leaves together after a timeout.
      bool ok = true;
      if constexpr (kTmaGate) ok = wait_or_abort(&s_g_full, n & 1, abort_flag);

      // ---- raw gate rows -> local cumulative sums; rows >= Cn contribute g = 0
      float G[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 4 * rg + u;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (r < Cn) {
          if constexpr (kGate == kGateLogTok) {
            a = make_float4(gtok[u], gtok[u], gtok[u], gtok[u]);
            b = a;
          } else if constexpr (kGate == kGateLogitBf16) {
            float x[8];
            tc::unpack8(*reinterpret_cast<const uint4*>(sm + FU_RAWG + r * 256 + 16 * co), x);
            a = make_float4(tc::neg_softplus_sfu(x[0]), tc::neg_softplus_sfu(x[1]), tc::neg_softplus_sfu(x[2]), tc::neg_softplus_sfu(x[3]));
            b = make_float4(tc::neg_softplus_sfu(x[4]), tc::neg_softplus_sfu(x[5]), tc::neg_softplus_sfu(x[6]), tc::neg_softplus_sfu(x[7]));
          } else {
            // the two 16-byte halves in alternating order across the quarter-warp (no bank conflicts)
            const float* gr = reinterpret_cast<const float*>(sm + FU_RAWG + r * 512) + c0;
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
        const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) G[u][e] = (u ? G[u - 1][e] : 0.f) + x[e];
      }
      // Row-group totals: this warp holds row groups 2w (lanes 0..15) and 2w+1
      // (lanes 16..31) of the same channels; the warp's total goes to s_wtot,
      // which lives over the raw gate rows once every thread has read its own.
      float lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = __shfl_xor_sync(0xffffffffu, G[3][e], 16);
      if (ptx::bar_or(1, 256, !ok || *abort_flag)) break;  // raw gate rows consumed
      if (lane >= 16) {
        reinterpret_cast<float4*>(s_wtot + warp * D + c0)[0] =
            make_float4(G[3][0] + lo[0], G[3][1] + lo[1], G[3][2] + lo[2], G[3][3] + lo[3]);
        reinterpret_cast<float4*>(s_wtot + warp * D + c0)[1] =
            make_float4(G[3][4] + lo[4], G[3][5] + lo[5], G[3][6] + lo[6], G[3][7] + lo[7]);
      }
      ptx::bar_sync(1, 256);  // warp totals visible
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
      // G is non-increasing (g <= 0): G at the chunk's last row is each channel's
      // minimum; G at the last row of blocks 0..2 are the block references.
      bool steep = false;
      if (rg == 15) {
        reinterpret_cast<float4*>(s_glast + c0)[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
        reinterpret_cast<float4*>(s_glast + c0)[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
#pragma unroll
        for (int e = 0; e < 8; ++e) steep |= !(G[3][e] >= tc::kChunkRefMinG);
      }
      if ((rg & 3) == 3 && rg < 15) {
        reinterpret_cast<float4*>(&s_gref[(rg + 1) >> 2][c0])[0] = make_float4(G[3][0], G[3][1], G[3][2], G[3][3]);
        reinterpret_cast<float4*>(&s_gref[(rg + 1) >> 2][c0])[1] = make_float4(G[3][4], G[3][5], G[3][6], G[3][7]);
      }
      // uniform over the group; s_glast, s_gref visible; s_wtot (the raw gate buffer) read
      const bool fast = !ptx::bar_or(1, 256, steep);
      if (fast && tid == 0) issue_g(n + 1, &g_issued);  // the raw gate buffer is free

      ok = wait_or_abort(&s_kq_full[s], (n >> 1) & 1, abort_flag);
      // K e^-G, gamma of this slot: the state is done with chunk n-2
      if (n >= 2) ok = ok && wait_or_abort(&s_rb_free[s], ((n - 2) >> 1) & 1, abort_flag);
      // 1 / |k_r| and 1 / |q_r| over dk (only when the call normalises), once k
      // and q have landed (the gate phase above overlaps their copy): the 16
      // lanes of a half-warp hold one row; k and q are read from their panels.
      if constexpr (kPrep) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * rg + u;
          float kx[8], qx[8];
          tc::unpack8(*reinterpret_cast<const uint4*>(l3 + kp * 16384 + ptx::sw128_chunk(r, ck)), kx);
          tc::unpack8(*reinterpret_cast<const uint4*>(l3 + kp * 16384 + 8192 + ptx::sw128_chunk(r, ck)), qx);
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
            s_nrm[0][r] = rsqrtf(fmaxf(sk, 1e-24f));
            s_nrm[1][r] = rsqrtf(fmaxf(sq, 1e-24f));
          }
        }
      }
      if (ptx::bar_or(1, 256, !ok || *abort_flag)) break;
      if (tid < C) s_beta[s][tid] = bt;  // the solver is done with chunk n-2's

      if (fast) {
        // Single reference (chunk start): a = e^{G} <= 1, rho = e^{-G} <= e^80.
        // Each 16-byte piece (8 channels of one row) is rewritten in place.
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * rg + u;
          uint8_t* pk = l3 + kp * 16384 + ptx::sw128_chunk(r, ck);
          uint8_t* pq = pk + 8192;
          uint4 kw = *reinterpret_cast<const uint4*>(pk), qw = *reinterpret_cast<const uint4*>(pq);
          if (r >= Cn) kw = qw = make_uint4(0u, 0u, 0u, 0u);
          const float nk = kPrep ? s_nrm[0][r] : 1.f, nq = kPrep ? s_nrm[1][r] : 1.f;
          uint32_t ka[4], qa[4], kr[4];
#pragma unroll
          for (int p2 = 0; p2 < 4; ++p2) {
            float2 kf = bf2(word(kw, p2)), qf = bf2(word(qw, p2));
            if constexpr (kPrep) {
              kf.x *= nk; kf.y *= nk;
              qf.x *= nq; qf.y *= nq;
            }
            const float t0 = G[u][2 * p2] * kLog2e, t1 = G[u][2 * p2 + 1] * kLog2e;  // in [-115.5, 0]
            const float a0 = ptx::ex2(t0), a1 = ptx::ex2(t1);
            ka[p2] = ptx::pack_bf16x2(kf.x * a0, kf.y * a1);
            qa[p2] = ptx::pack_bf16x2(qf.x * a0, qf.y * a1);
            kr[p2] = ptx::pack_bf16x2(kf.x * ptx::ex2(-t0), kf.y * ptx::ex2(-t1));
          }
          *reinterpret_cast<uint4*>(pk) = make_uint4(ka[0], ka[1], ka[2], ka[3]);
          *reinterpret_cast<uint4*>(pq) = make_uint4(qa[0], qa[1], qa[2], qa[3]);
          *reinterpret_cast<uint4*>(rb + kp * 8192 + ptx::sw128_chunk(r, ck)) = make_uint4(kr[0], kr[1], kr[2], kr[3]);
        }
      } else {
        // Steep chunk: some channel decays by more than 80 over the chunk.  [A'; P']
        // is accumulated from four MMAs, one per 16-row block I, with the block's
        // reference rho_I = G at the end of block I-1 (0 for I = 0): left rows of
        // block I scaled by e^{G - rho_I} <= 1 (other rows zero), right rows
        // j <= end of block I scaled by e^{rho_I - G_j} (<= e^80 inside block I,
        // <= 1 before it; later rows zero).  The left operand sits over the raw
        // gate rows, whose next load waits until the four MMAs are done.
        if (tid == 0 && n >= 2) wait_or_abort(&s_s_ready[s], ((n - 2) >> 1) & 1, abort_flag);
        uint8_t* lft = sm + FU_RAWG;
        bool quit = false;
        for (int I = 0; I < 4; ++I) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = 4 * rg + u, blk = rg >> 2;
            uint4 kw = *reinterpret_cast<const uint4*>(l3 + kp * 16384 + ptx::sw128_chunk(r, ck));
            uint4 qw = *reinterpret_cast<const uint4*>(l3 + kp * 16384 + 8192 + ptx::sw128_chunk(r, ck));
            if (r >= Cn) kw = qw = make_uint4(0u, 0u, 0u, 0u);
            const float nk = kPrep ? s_nrm[0][r] : 1.f, nq = kPrep ? s_nrm[1][r] : 1.f;
            uint32_t lk[4], lq[4], rr[4];
#pragma unroll
            for (int p2 = 0; p2 < 4; ++p2) {
              float2 kf = bf2(word(kw, p2)), qf = bf2(word(qw, p2));
              if constexpr (kPrep) {
                kf.x *= nk; kf.y *= nk;
                qf.x *= nq; qf.y *= nq;
              }
              const float2 ref = I ? *reinterpret_cast<const float2*>(&s_gref[I][c0 + 2 * p2]) : make_float2(0.f, 0.f);
              // d <= 0 for rows in or after block I, >= 0 before it
              const float d0 = (G[u][2 * p2] - ref.x) * kLog2e, d1 = (G[u][2 * p2 + 1] - ref.y) * kLog2e;
              const float a0 = blk == I ? ptx::ex2(d0) : 0.f, a1 = blk == I ? ptx::ex2(d1) : 0.f;
              lk[p2] = ptx::pack_bf16x2(kf.x * a0, kf.y * a1);
              lq[p2] = ptx::pack_bf16x2(qf.x * a0, qf.y * a1);
              rr[p2] = blk <= I ? ptx::pack_bf16x2(kf.x * ptx::ex2(-d0), kf.y * ptx::ex2(-d1)) : 0u;
            }
            *reinterpret_cast<uint4*>(lft + kp * 16384 + ptx::sw128_chunk(r, ck)) = make_uint4(lk[0], lk[1], lk[2], lk[3]);
            *reinterpret_cast<uint4*>(lft + kp * 16384 + ptx::sw128_chunk(64 + r, ck)) =
                make_uint4(lq[0], lq[1], lq[2], lq[3]);
            *reinterpret_cast<uint4*>(rb + kp * 8192 + ptx::sw128_chunk(r, ck)) = make_uint4(rr[0], rr[1], rr[2], rr[3]);
          }
          ptx::fence_proxy_async_smem();
          if (ptx::bar_or(1, 256, *abort_flag != 0)) {
            quit = true;
            break;
          }
          if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t id = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t ad = ptx::sdesc_sw128(sb + FU_RAWG + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = ptx::sdesc_sw128(sb + FU_RB + s * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
              ptx::mma_bf16(tmem + 64 * s, ad, bd, id, (I > 0 || kk > 0) ? 1u : 0u);
            }
            mma_issued = true;
            ptx::mma_commit(&s_st);
          }
          // the operands are rewritten by the next round: wait for this MMA
          wait_or_abort(&s_st, st_round & 1, abort_flag);
          ++st_round;
        }
        if (quit || ptx::bar_or(1, 256, *abort_flag != 0)) break;
        // the state's operands: K e^G, Q e^G (chunk start, in place), Kbar = K e^{G_last - G}
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * rg + u;
          uint8_t* pk = l3 + kp * 16384 + ptx::sw128_chunk(r, ck);
          uint8_t* pq = pk + 8192;
          uint4 kw = *reinterpret_cast<const uint4*>(pk), qw = *reinterpret_cast<const uint4*>(pq);
          if (r >= Cn) kw = qw = make_uint4(0u, 0u, 0u, 0u);
          const float nk = kPrep ? s_nrm[0][r] : 1.f, nq = kPrep ? s_nrm[1][r] : 1.f;
          uint32_t ka[4], qa[4], kb[4];
#pragma unroll
          for (int p2 = 0; p2 < 4; ++p2) {
            float2 kf = bf2(word(kw, p2)), qf = bf2(word(qw, p2));
            if constexpr (kPrep) {
              kf.x *= nk; kf.y *= nk;
              qf.x *= nq; qf.y *= nq;
            }
            const float2 gl2 = *reinterpret_cast<const float2*>(&s_glast[c0 + 2 * p2]);
            const float a0 = ptx::ex2(G[u][2 * p2] * kLog2e), a1 = ptx::ex2(G[u][2 * p2 + 1] * kLog2e);
            ka[p2] = ptx::pack_bf16x2(kf.x * a0, kf.y * a1);
            qa[p2] = ptx::pack_bf16x2(qf.x * a0, qf.y * a1);
            kb[p2] = ptx::pack_bf16x2(kf.x * ptx::ex2((gl2.x - G[u][2 * p2]) * kLog2e),
                                      kf.y * ptx::ex2((gl2.y - G[u][2 * p2 + 1]) * kLog2e));
          }
          *reinterpret_cast<uint4*>(pk) = make_uint4(ka[0], ka[1], ka[2], ka[3]);
          *reinterpret_cast<uint4*>(pq) = make_uint4(qa[0], qa[1], qa[2], qa[3]);
          *reinterpret_cast<uint4*>(rb + kp * 8192 + ptx::sw128_chunk(r, ck)) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
        }
      }
      if (rg == 0) {
        float gm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) gm[e] = expf(s_glast[c0 + e]);
        float* gam = reinterpret_cast<float*>(sm + FU_GAM + (n & 3) * 512);
        reinterpret_cast<float4*>(gam)[2 * co] = make_float4(gm[0], gm[1], gm[2], gm[3]);
        reinterpret_cast<float4*>(gam)[2 * co + 1] = make_float4(gm[4], gm[5], gm[6], gm[7]);
      }
      if (tid == 0 && !fast) s_ring[n & 7].flags |= kItSteep;
      ptx::fence_proxy_async_smem();
      ptx::bar_sync(1, 256);  // operands, s_beta[s], gamma complete

      if (tid == 0) {
        if (fast) {
          // TMEM slot s: the solver is done with chunk n-2
          const bool go = !*abort_flag && (n < 2 || wait_or_abort(&s_s_ready[s], ((n - 2) >> 1) & 1, abort_flag));
          if (go) {
            // [A'; P'] = [K e^G; Q e^G] (K e^-G)^T : M=128, N=64, K=128
            ptx::tc_fence_after();
            constexpr uint32_t id = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t ad = ptx::sdesc_sw128(sb + FU_L3 + s * FU_L3_SLOT + (kk >> 2) * 16384 + (kk & 3) * 32,
                                                   16, 1024);
              const uint64_t bd = ptx::sdesc_sw128(sb + FU_RB + s * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
              ptx::mma_bf16(tmem + 64 * s, ad, bd, id, kk > 0);
            }
            mma_issued = true;
            ptx::mma_commit(&s_a_done[s]);
          } else {
            ptx::mbar_arrive(&s_a_done[s]);
          }
        } else {
          ptx::mbar_arrive(&s_a_done[s]);  // the block MMAs have completed already
          issue_g(n + 1, &g_issued);       // the raw gate buffer is free again
        }
        ptx::mbar_arrive(&s_a_done[s]);  // releases s_beta[s] and the descriptor's flags
      }
    }
  } else if (warp < 16) {
    // ============================== solver ==============================
    const int st = tid - 256, w8 = warp - 8;
    const int qd = warp & 3, ch = w8 >> 2;  // TMEM lane quarter; 32-column half
    float* As = reinterpret_cast<float*>(sm + FU_AS);
    constexpr int kVIssuer = 224;  // warp 7 of the group: idle in the middle of the solve
    if (st == kVIssuer) {
      ptx::prefetch_tmap(&tm_v);
      issue_v(0, v_issued);
    }
    uint32_t real = 0;  // chunks solved (phases of uw_done and of the state's x_free)
    for (uint32_t n = 0;; ++n) {
      const int s = n & 1;
      bool ok = wait_or_abort(&s_a_done[s], (n >> 1) & 1, abort_flag);
      // P of this slot: the state is done with chunk n-2's P and output tile
      if (n >= 2) ok = ok && wait_or_abort(&s_p_free[s], ((n - 2) >> 1) & 1, abort_flag);
      if (ptx::bar_or(2, 256, !ok || *abort_flag)) break;  // uniform over the group
      ptx::tc_fence_after();
      const FuItem it = s_ring[n & 7];
      if (!(it.flags & (kItEnd | kItEmpty))) {
        uint8_t* l3 = sm + FU_L3 + s * FU_L3_SLOT;
        // scatter A (fp32, beta-scaled) and P (bf16) out of TMEM slot s
        const bool big =
            tc::scatter_single_ref(tmem + 64 * s, s_beta[s], As, sm + FU_P + s * 8192, warp, w8, lane, false);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        const bool accurate = ptx::bar_or(2, 256, big);
        // the plain instance leaves such a chunk to the precise one: it marks the unit
        if (!kPrecise && accurate && st == 0) s_doom[it.ord & 3] = 1;
        // T = (I + A)^{-1} over A, T diag(beta) as bf16 hi (FU_TT), and for a chunk
        // with near-parallel keys also its lo part (FU_TLO).  V of chunk n+1 goes
        // into the other slot (its V, chunk n-1's, is read) from the warp that is
        // idle at that point of the solve.
        auto sync2 = [] { ptx::bar_sync(2, 256); };
        auto idle = [&] {
          if (lane == 0) issue_v(n + 1, v_issued);
        };
        if (kPrecise && accurate)
          tc::solve_t_beta_precise(As, s_beta[s], sm + FU_TT, sm + FU_TLO, st, w8, lane, sync2, idle);
        else
          tc::solve_t_beta<false>(As, s_beta[s], sm + FU_TT, nullptr, st, w8, lane, sync2, idle);
        ptx::fence_proxy_async_smem();
        ptx::bar_sync(2, 256);
        // ---- W^T = (K e^G)^T (T diag(beta))^T into TMEM slot s (free since the
        //      scatter), U^T = V^T (T diag(beta))^T into the state's X^T columns
        //      (free once the state has split chunk n-1's E): M=128, N=64, K=64,
        //      T diag(beta) as hi, then (near-parallel keys) lo.
        if (st == 0) {
          bool go = wait_or_abort(&s_v_full[s], (n >> 1) & 1, abort_flag);
          go = go && (real == 0 || wait_or_abort(&s_x_free, (real - 1) & 1, abort_flag));
          if (go) {
            ptx::tc_fence_after();
            constexpr uint32_t id = ptx::idesc_bf16(128, 64, true, false);
            const uint32_t kg = sb + FU_L3 + s * FU_L3_SLOT, vs = sb + FU_V + s * 16384;
            const int parts = kPrecise && accurate ? 2 : 1;
#pragma unroll 1
            for (int part = 0; part < parts; ++part) {
              const uint32_t tb = sb + (part ? FU_TLO : FU_TT);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                ptx::mma_bf16(tmem + 64 * s, ptx::sdesc_sw128(kg + i * 2048, 16384, 1024),
                              ptx::sdesc_sw128(tb + i * 32, 16, 1024), id, (part | i) > 0);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                ptx::mma_bf16(tmem + kTmX, ptx::sdesc_sw128(vs + i * 2048, 8192, 1024),
                              ptx::sdesc_sw128(tb + i * 32, 16, 1024), id, (part | i) > 0);
            }
            mma_issued = true;
            ptx::mma_commit(&s_uw_done);
          } else {
            ptx::mbar_arrive(&s_uw_done);
          }
        }
        ok = wait_or_abort(&s_uw_done, real & 1, abort_flag);
        ptx::tc_fence_after();
        // ---- -W (bf16) over the K e^G rows of the slot, in their layout (K-major:
        //      row = token, key channels 0..63 | 64..127 in the two panels), so that
        //      the state's first MMA reads [-W; Q e^G] as one 128-row operand
        store_tile_t(tmem + ((uint32_t)(32 * qd) << 16) + 64 * s + 32 * ch, ptx::smem_u32(l3), 32 * qd, 32 * ch,
                     16384, -1.f, lane);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        if (ptx::bar_or(2, 256, !ok || *abort_flag)) break;
        ++real;
      } else if (st == kVIssuer) {  // keep V's per-chunk phases in step
        issue_v(n + 1, v_issued);
      }
      if (st == 0) ptx::mbar_arrive(&s_s_ready[s]);
      if (it.flags & kItEnd) break;
    }
  } else {
    // ============================== state ==============================
    const int st = tid - 512, qd = warp & 3;
    const int dv = 32 * qd + lane;  // this thread's value channel = its TMEM lane
    const uint32_t lo_lane = (uint32_t)(32 * qd) << 16;
    if (st == 0) {
      issue_kq(0, kq_issued);
      issue_kq(1, kq_issued);
    }
    zero_cols64(tmem + lo_lane + kTmO);  // the first MMA accumulates O onto zeros
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    // chunk m's output tile is read by its tensor stores (issued by this thread):
    // the tile's P slot and the 8 KB panel are free
    auto release_tile = [&](uint32_t m) {
      ptx::bulk_wait_read0();
      ptx::mbar_arrive(&s_p_free[m & 1]);
    };
    uint32_t real = 0;  // chunks with MMAs (phases of m1, m3, x_free)
    for (uint32_t n = 0;; ++n) {
      const int s = n & 1;
      const bool okr = wait_or_abort(&s_s_ready[s], (n >> 1) & 1, abort_flag);
      if (ptx::bar_or(3, 128, !okr || *abort_flag)) break;  // uniform over the group
      ptx::tc_fence_after();
      const FuItem it = s_ring[n & 7];
      if (it.flags & kItEnd) break;
      const size_t urow = (size_t)it.unit * D;  // first state row of the unit
      if (it.flags & kItEmpty) {  // an empty sequence hands its initial state through
        if (S_out)
          for (int c = 0; c < D; ++c) S_out[(urow + c) * D + dv] = S0 ? S0[(urow + c) * D + dv] : 0.f;
        if (st == 0) {  // keep the per-chunk phases in step
          if (n >= 1) release_tile(n - 1);
          issue_kq(n + 2, kq_issued);
          ptx::mbar_arrive(&s_rb_free[s]);
        }
        continue;
      }
      const bool steep = (it.flags & kItSteep) != 0;
      if (it.flags & kItFirst) {  // the unit's initial state, transposed: row dv of S^T
#pragma unroll 1
        for (int c16 = 0; c16 < D; c16 += 16) {
          float x[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] = S0 ? S0[(urow + c16 + e) * D + dv] : 0.f;
          ptx::tmem_st16(tmem + lo_lane + kTmS + c16, x);
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = ptx::pack_bf16x2(x[2 * i], x[2 * i + 1]);
          ptx::tmem_st8u(tmem + lo_lane + kTmSb + c16 / 2, w);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::bar_sync(3, 128);
      }
      // ---- [E^T | (Q e^G S)^T] = [U^T | 0] + S^T [-W; Q e^G]^T  (N=128, K=128: the
      //      slot's panel rows are -W (tokens 0..63) and Q e^G (64..127), K-major;
      //      the E half accumulates onto the solver's U^T, the other onto zeros)
      if (st == 0) {
        ptx::tc_fence_after();
        constexpr uint32_t id = ptx::idesc_bf16(128, 128, false, false);
        const uint32_t l3s = sb + FU_L3 + s * FU_L3_SLOT;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_ts(tmem + kTmX, tmem + kTmSb + 8 * kk,
                           ptx::sdesc_sw128(l3s + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), id, 1);
        mma_issued = true;
        ptx::mma_commit(&s_m1);
        if (n >= 1) release_tile(n - 1);  // while the MMAs run
      }
      const float* gam = reinterpret_cast<const float*>(sm + FU_GAM + (n & 3) * 512);
      if (steep) {  // Kbar form: decay the state first (the MMAs above read only the bf16 copy)
#pragma unroll 1
        for (int c32 = 0; c32 < D; c32 += 32) {
          float x[32];
          ld32(tmem + lo_lane + kTmS + c32, x);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= gam[c32 + e];
          ptx::tmem_st16(tmem + lo_lane + kTmS + c32, *reinterpret_cast<float(*)[16]>(x));
          ptx::tmem_st16(tmem + lo_lane + kTmS + c32 + 16, *reinterpret_cast<float(*)[16]>(x + 16));
        }
      }
      bool ok = wait_or_abort(&s_m1, real & 1, abort_flag);
      ptx::tc_fence_after();
      // the slot's panels are read: chunk n+2's k, q may land.  Thread 0 arms the
      // barrier now; after the group barrier below each warp's lane 0 issues one
      // of the four tensor copies, so that no thread issues all four.
      if (st == 0) s_kq_mode = arm_kq(n + 2, kq_issued);
      // ---- E (fp32) as bf16 hi | lo
#pragma unroll 1
      for (int h2 = 0; h2 < 2; ++h2) {
        float x[32];
        ld32(tmem + lo_lane + kTmX + 32 * h2, x);
        ptx::tmem_wait_ld();
        store_hi_lo32(tmem + lo_lane + kTmHL, h2, x);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      if (ptx::bar_or(3, 128, !ok || *abort_flag)) break;
      if (lane == 0 && s_kq_mode) issue_kq_part(n + 2, qd);
      if (st == 0) {
        ptx::mbar_arrive(&s_x_free);  // E^T's columns are read: the next U^T may land there
        ptx::tc_fence_after();
        // S^T += E^T (K e^-G) (Kbar for a steep chunk): N=128, K=64, B MN-major
        constexpr uint32_t id2 = ptx::idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          ptx::mma_bf16_ts(tmem + kTmS, tmem + kTmHL + (i >> 2) * 32 + 8 * (i & 3),
                           ptx::sdesc_sw128(sb + FU_RB + s * 16384 + (i & 3) * 2048, 8192, 1024), id2, 1);
        // (Q e^G S)^T += E^T P^T: N=64, K=64, B K-major
        constexpr uint32_t id3 = ptx::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          ptx::mma_bf16_ts(tmem + kTmO, tmem + kTmHL + (i >> 2) * 32 + 8 * (i & 3),
                           ptx::sdesc_sw128(sb + FU_P + s * 8192 + (i & 3) * 32, 16, 1024), id3, 1);
        ptx::mma_commit(&s_m3);
      }
      ok = wait_or_abort(&s_m3, real & 1, abort_flag);
      if (ptx::bar_or(3, 128, !ok || *abort_flag)) break;
      ptx::tc_fence_after();
      // K e^-G and P of this slot are read; gamma has a slot of its own per chunk mod 4
      if (st == 0) ptx::mbar_arrive(&s_rb_free[s]);
      // ---- decay (single-reference chunks), the next chunk's bf16 operand, the outputs
#pragma unroll 1
      for (int c32 = 0; c32 < D; c32 += 32) {
        float x[32];
        ld32(tmem + lo_lane + kTmS + c32, x);
        ptx::tmem_wait_ld();
        if (!steep) {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= gam[c32 + e];
          ptx::tmem_st16(tmem + lo_lane + kTmS + c32, *reinterpret_cast<float(*)[16]>(x));
          ptx::tmem_st16(tmem + lo_lane + kTmS + c32 + 16, *reinterpret_cast<float(*)[16]>(x + 16));
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = ptx::pack_bf16x2(x[2 * i], x[2 * i + 1]);
        ptx::tmem_st16u(tmem + lo_lane + kTmSb + c32 / 2, w);
      }
      // the output tile, two 64-channel panels [64 tokens][128 B], 128-byte
      // swizzled: value channels 0..63 over this slot's P (read by the MMAs
      // above), 64..127 in FU_OST (read by chunk n-1's store)
      uint8_t* opan[2] = {sm + FU_P + s * 8192, sm + FU_OST};
#pragma unroll 1
      for (int h2 = 0; h2 < 2; ++h2)
        store_tile_t(tmem + lo_lane + kTmO + 32 * h2, ptx::smem_u32(opan[qd >> 1]), 32 * (qd & 1), 32 * h2, 0, 1.f,
                     lane);
      zero_cols64(tmem + lo_lane + kTmO);  // the next chunk's first MMA accumulates O onto zeros
      // plain instance, the unit's last chunk: a unit that met near-parallel keys
      // is left to the precise instance (its state is not written, so an S_out
      // aliasing S0 keeps S0; its output rows are written again)
      const bool doomed = !kPrecise && (it.flags & kItLast) && s_doom[it.ord & 3] != 0;
      ptx::fence_proxy_async_smem();
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::bar_sync(3, 128);  // every read of X^T done; tile complete
      if (doomed && st == 0) {
        s_doom[it.ord & 3] = 0;
        unit_mark[it.unit] = 1;
        *any_mark = 1;
      }
      const int h = it.unit % H;
      if (it.Cn == C) {  // a whole chunk: two tensor stores
        if (st == 0) {
          ptx::tma_store_3d(&tm_o, 0, h, (int)it.s0, opan[0]);
          ptx::tma_store_3d(&tm_o, 64, h, (int)it.s0, opan[1]);
          ptx::bulk_commit();
        }
      } else {  // the ragged last chunk of a sequence: 16-byte pieces of its rows
#pragma unroll 1
        for (int piece = st; piece < C * 16; piece += 128) {
          const int r = piece >> 4, c16 = piece & 15;
          if (r < it.Cn) {
            const uint4 val =
                *reinterpret_cast<const uint4*>(opan[c16 >> 3] + r * 128 + ((((c16 & 7) ^ r) & 7) << 4));
            *reinterpret_cast<uint4*>(o + ((size_t)(it.s0 + r) * H + h) * D + 8 * c16) = val;
          }
        }
        ptx::bar_sync(3, 128);  // the tile is read
      }
      if ((it.flags & kItLast) && S_out && !doomed) {
#pragma unroll 1
        for (int c32 = 0; c32 < D; c32 += 32) {
          float x[32];
          ld32(tmem + lo_lane + kTmS + c32, x);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) S_out[(urow + c32 + e) * D + dv] = x[e];
        }
      }
      ++real;
    }
    if (st == 0) ptx::bulk_wait0();  // the output tiles have landed
  }

  // After a timeout: wait (bounded again) for the copies and MMAs still in
  // flight, so that nothing lands in shared or tensor memory after exit.
  ptx::tc_fence_before();
  __syncthreads();
  if (s_abort) {
    if (tid == 0 && g_issued) ptx::mbar_wait_bounded(&s_g_full, (g_issued - 1) & 1, 1000000000ull);
    if (tid == 512)
      for (int i = 0; i < 2; ++i)
        if (kq_issued[i]) ptx::mbar_wait_bounded(&s_kq_full[i], (kq_issued[i] - 1) & 1, 1000000000ull);
    if (tid == 256 + 224)
      for (int i = 0; i < 2; ++i)
        if (v_issued[i]) ptx::mbar_wait_bounded(&s_v_full[i], (v_issued[i] - 1) & 1, 1000000000ull);
  }
  if (s_abort && (tid == 0 || tid == 256 || tid == 512)) {  // the three MMA-issuing threads
    if (mma_issued) ptx::mma_commit(&s_drain);
    else ptx::mbar_arrive(&s_drain);
    ptx::mbar_wait_bounded(&s_drain, 0, 1000000000ull);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmCols);
}

// Set-up of one call (one CTA of 1024 threads): zeroes the unit counters, the
// unit marks (and, when the two-kernel path runs the precise instance as its
// fallback, the flag its chunk-local kernels raise) and,
// for packed sequences, checks cu_seqlens (cu[0] == 0, non-decreasing,
// cu[num_seqs] == T) -- a bad table raises the device error word and sets
// *status = -1, so the prefill kernel does nothing -- then orders the
// sequences longest first (rank by length, ties by index) when there are at
// most kSortMax of them; longer lists keep their order.
constexpr int kSortMax = 2048;
__global__ void __launch_bounds__(1024)
    kda_fused_setup_kernel(const int32_t* __restrict__ cu_seqlens, int num_seqs, int T, int* __restrict__ ctr,
                           int* __restrict__ status, int* __restrict__ order, int* __restrict__ esc_flag,
                           int* __restrict__ unit_mark, int units) {
  __shared__ int s_len[kSortMax];
  const int tid = threadIdx.x;
  if (tid == 0) {
    ctr[0] = ctr[1] = ctr[2] = 0;  // the plain and precise instances' unit counters, the any-unit mark
    if (esc_flag) *esc_flag = 0;
  }
  for (int i = tid; i < units; i += 1024) unit_mark[i] = 0;
  if (!cu_seqlens) return;
  bool bad = tid == 0 && (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T);
  for (int i = tid; i < num_seqs; i += 1024) bad |= cu_seqlens[i + 1] < cu_seqlens[i];
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      raise_device_error(kDevErrBadSeqlens);
      *status = -1;
    }
    return;
  }
  if (tid == 0) *status = 0;
  if (num_seqs > kSortMax) {
    for (int i = tid; i < num_seqs; i += 1024) order[i] = i;
    return;
  }
  for (int i = tid; i < num_seqs; i += 1024) s_len[i] = cu_seqlens[i + 1] - cu_seqlens[i];
  __syncthreads();
  for (int i = tid; i < num_seqs; i += 1024) {
    const int li = s_len[i];
    int rank = 0;
    for (int j = 0; j < num_seqs; ++j) {
      const int lj = s_len[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
// Workspace: the plain and precise instances' unit counters, the any-unit
// mark, the table check's status (ints 0..3), the sequence order (from byte
// 256), then one mark per (sequence, head) unit.
inline size_t fused_workspace_bytes(int num_seqs, long long units) {
  return 256 + ((size_t)std::max(num_seqs, 0) + (size_t)std::max(units, 0LL)) * sizeof(int);
}

inline bool fused_kernel_available() {
  static PerDeviceOnce once;
  static bool ok[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  run_once_per_device(once, [dev] {
    const void* fns[] = {
#define KDA_FU_FN(M) (const void*)kda_fused_prefill_kernel<M, false, false>,                                      \
                     (const void*)kda_fused_prefill_kernel<M, true, false>,                                       \
                     (const void*)kda_fused_prefill_kernel<M, false, true>,                                       \
                     (const void*)kda_fused_prefill_kernel<M, true, true>
        KDA_FU_FN(kGateLogCh), KDA_FU_FN(kGateLogTok), KDA_FU_FN(kGateLogitF32), KDA_FU_FN(kGateLogitBf16)
#undef KDA_FU_FN
    };
    int optin = 0;
    bool all = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess;
    for (const void* fn : fns) {
      cudaFuncAttributes fa{};
      all = all && cudaFuncGetAttributes(&fa, fn) == cudaSuccess &&
            (size_t)FU_DYN + fa.sharedSizeBytes <= (size_t)optin &&
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FU_DYN) == cudaSuccess;
    }
    ok[dev] = all;
    cudaGetLastError();  // an unavailable kernel is not an error of the call
    return cudaSuccess;
  });
  return ok[dev];
}

// Launches the set-up kernel (phase & kFusedSetup), the plain instance of the
// prefill kernel (phase & kFusedMain) and its precise instance (phase &
// kFusedPrecise).  After the plain instance, the precise one recomputes only
// the units the plain one marked (those with a chunk of near-parallel keys)
// and returns at once when there are none.  With esc_flag the set-up kernel
// and the precise instance are the two-kernel path's precise fallback: the
// set-up kernel zeroes *esc_flag, and the precise instance (launched after the
// state pass) recomputes the whole call only if a chunk-local kernel raised it.
constexpr int kFusedSetup = 1, kFusedMain = 2, kFusedPrecise = 4;
template <int kGate>
inline cudaError_t launch_fused_t(const bf16* q, const bf16* k, const bf16* v, const void* g, const float* beta,
                                  const float* S0, bf16* o, float* S_out, const int32_t* cu_seqlens, int N,
                                  int B, int T, int H, void* workspace, int sms, cudaStream_t stream,
                                  int phase, int* esc_flag) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  cudaError_t e = ws::tensor_map_encoder(&enc);
  if (e != cudaSuccess) return e;
  const long long tokens = (long long)B * T;
  CUtensorMap mk, mq, mg, mv, mo;
  if ((e = ws::encode_rows_map(enc, &mo, o, false, tokens, H, 64, true)) != cudaSuccess) return e;
  if ((e = ws::encode_rows_map(enc, &mk, k, false, tokens, H, 64, true)) != cudaSuccess) return e;
  if ((e = ws::encode_rows_map(enc, &mq, q, false, tokens, H, 64, true)) != cudaSuccess) return e;
  if ((e = ws::encode_rows_map(enc, &mv, v, false, tokens, H, 64, true)) != cudaSuccess) return e;
  if constexpr (kGate == kGateLogTok) {
    mg = mk;  // not read: a per-token gate takes plain loads
  } else {
    if ((e = ws::encode_rows_map(enc, &mg, g, kGate != kGateLogitBf16, tokens, H, D, false)) != cudaSuccess) return e;
  }
  const long long units = (long long)N * H;
  int* wsi = static_cast<int*>(workspace);
  int* ctr_plain = wsi;
  int* ctr_precise = wsi + 1;
  int* any_mark = wsi + 2;
  int* status = wsi + 3;
  int* order = wsi + 64;
  int* marks = wsi + 64 + (cu_seqlens ? N : 0);
  if (phase & kFusedSetup) {
    kda_fused_setup_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, cu_seqlens ? N : 0, T, ctr_plain, status, order,
                                                   esc_flag, marks, (int)units);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int grid = (int)std::min<long long>(units, sms);
  if (grid <= 0) return cudaSuccess;
  const int* ord = cu_seqlens ? order : nullptr;
  if (phase & kFusedMain) {
    if (cu_seqlens)
      kda_fused_prefill_kernel<kGate, true, false><<<grid, kThreads, FU_DYN, stream>>>(
          mk, mq, mg, mv, mo, g, beta, S0, o, S_out, cu_seqlens, N, T, H, ctr_plain, ord, status, nullptr, marks,
          any_mark);
    else
      kda_fused_prefill_kernel<kGate, false, false><<<grid, kThreads, FU_DYN, stream>>>(
          mk, mq, mg, mv, mo, g, beta, S0, o, S_out, nullptr, N, T, H, ctr_plain, ord, status, nullptr, marks,
          any_mark);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (phase & kFusedPrecise) {
    // after the plain instance: its marked units; as the two-kernel fallback: all
    const int* gate_flag = esc_flag ? esc_flag : any_mark;
    int* filter = esc_flag ? nullptr : marks;
    if (cu_seqlens)
      kda_fused_prefill_kernel<kGate, true, true><<<grid, kThreads, FU_DYN, stream>>>(
          mk, mq, mg, mv, mo, g, beta, S0, o, S_out, cu_seqlens, N, T, H, ctr_precise, ord, status, gate_flag,
          filter, any_mark);
    else
      kda_fused_prefill_kernel<kGate, false, true><<<grid, kThreads, FU_DYN, stream>>>(
          mk, mq, mg, mv, mo, g, beta, S0, o, S_out, nullptr, N, T, H, ctr_precise, ord, status, gate_flag,
          filter, any_mark);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

inline cudaError_t launch_fused(const bf16* q, const bf16* k, const bf16* v, const void* g, const float* beta,
                                const float* S0, bf16* o, float* S_out, const int32_t* cu_seqlens, int N, int B,
                                int T, int H, void* workspace, int sms, int gmode, cudaStream_t stream,
                                int phase = kFusedSetup | kFusedMain | kFusedPrecise, int* esc_flag = nullptr) {
#define KDA_FU_CASE(M)                                                                                          \
  case M:                                                                                                       \
    return launch_fused_t<M>(q, k, v, g, beta, S0, o, S_out, cu_seqlens, N, B, T, H, workspace, sms, stream, \
                             phase, esc_flag)
  switch (gmode) {
    KDA_FU_CASE(kGateLogCh);
    KDA_FU_CASE(kGateLogTok);
    KDA_FU_CASE(kGateLogitF32);
    KDA_FU_CASE(kGateLogitBf16);
    default:
      return cudaErrorInvalidValue;
  }
#undef KDA_FU_CASE
}

}  // namespace fu
}  // namespace kda
