// kda_api.cu -- the C ABI of libkda (declared in include/kda.h): argument
// validation, workspace sizing, dispatch to the kernels, error reporting.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/kda.h"
#include "kda_chunk_bwd.cuh"
#include "kda_chunk_simt.cuh"
#include "kda_chunk_tc.cuh"
#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_host.cuh"

namespace {

thread_local char t_err[512] = "";
thread_local cudaEvent_t* t_prof_events = nullptr;
thread_local int t_prof_count = 0;
thread_local int t_seg_force = 0;  // kda_set_segment_chunks: 0 auto, > 0 fixed, < 0 never
thread_local int t_local_kernel = 0;  // kda_set_local_kernel: 0 default, 1 two-CTA kernel only
thread_local int t_prefill_path = 0;  // kda_set_prefill_path: 0 automatic, 1 single pass, 2 two kernels

int current_sms() { return kda::current_sm_count(); }

kda_status_t fail(kda_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return st;
}

kda_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(KDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1u)) == 0; }

bool supported_head(int dk, int dv) { return dk == dv && (dk == 32 || dk == 64 || dk == 128); }

bool use_tensor_core_path(int dk, int dv, int chunk_size, kda_dtype_t dt) {
  return kda::kTcPathBuilt && dt == KDA_BF16 && dk == 128 && dv == 128 && chunk_size == 64;
}

long long max_chunks(int B, int T, int num_seqs, int chunk_size) {
  if (num_seqs > 0) return (long long)T / chunk_size + num_seqs;
  return (long long)B * ((T + chunk_size - 1) / chunk_size);
}

// The tensor-core prefill's choices for these sizes on the current device and
// this thread's settings: sequence segments (two-kernel path only) and the path.
struct TcPlan {
  int seg;
  bool fused;
};
TcPlan tc_plan(int B, int T, int H, int num_seqs) {
  const int sms = current_sms();
  TcPlan p;
  p.seg = kda::tc_segment_chunks(B, T, H, num_seqs, sms, t_seg_force);
  p.fused = kda::tc_use_fused(B, T, H, num_seqs, sms, t_prefill_path == kda::kPathFused ? 0 : p.seg,
                              t_prefill_path) &&
            kda::fu::fused_kernel_available();
  if (p.fused) p.seg = 0;
  return p;
}

template <typename TIn>
cudaError_t dispatch_chunk_simt(int dk, int C, const void* q, const void* k, const void* v,
                                const void* g, const float* beta, const float* S0, void* o,
                                float* S_out, const int32_t* cu, int N, int T, int H, int dv,
                                int gmode, cudaStream_t st) {
#define KDA_SIMT_CASE(D, CC)                                                                  \
  if (dk == D && C == CC)                                                                     \
    return kda::launch_chunk_simt<TIn, D, CC>(q, k, v, g, beta, S0, o, S_out, cu, N, T, H, dv, \
                                               gmode, st);
  KDA_SIMT_CASE(32, 16) KDA_SIMT_CASE(32, 32) KDA_SIMT_CASE(32, 64)
  KDA_SIMT_CASE(64, 16) KDA_SIMT_CASE(64, 32) KDA_SIMT_CASE(64, 64)
  KDA_SIMT_CASE(128, 16) KDA_SIMT_CASE(128, 32) KDA_SIMT_CASE(128, 64)
#undef KDA_SIMT_CASE
  return cudaErrorInvalidValue;
}

template <typename TIn>
cudaError_t dispatch_decode(int dk, const void* q, const void* k, const void* v, const void* g,
                            const float* beta, float* S, void* o, int N, int H, int gmode,
                            cudaStream_t st) {
  if (dk == 32) return kda::launch_decode_step<TIn, 32, 32>(q, k, v, g, beta, S, o, N, H, gmode, st);
  if (dk == 64) return kda::launch_decode_step<TIn, 64, 64>(q, k, v, g, beta, S, o, N, H, gmode, st);
  if (dk == 128) return kda::launch_decode_step<TIn, 128, 128>(q, k, v, g, beta, S, o, N, H, gmode, st);
  return cudaErrorInvalidValue;
}

// gmode (kda::GateMode): g holds log alpha per key channel ([.., H, dk], KDA)
// or per token and head ([.., H], Gated DeltaNet), or raw per-channel logits
// (fp32 or bf16) with q, k normalised and beta given as a logit.
kda_status_t chunk_fwd_impl(const char* fn, const void* q, const void* k, const void* v,
                            const void* g, const float* beta, const float* S0, void* o,
                            float* S_out, const int32_t* cu_seqlens, int num_seqs, int B, int T,
                            int H, int dk, int dv, int chunk_size, kda_dtype_t dtype,
                            void* workspace, size_t workspace_bytes, int gmode,
                            cudaStream_t stream) {
  t_err[0] = 0;
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0)
    return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d num_seqs=%d", fn, B,
                T, H, num_seqs);
  if (dtype != KDA_BF16 && dtype != KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dtype);
  if (!supported_head(dk, dv))
    return fail(KDA_ERR_UNSUPPORTED, "%s: dk=%d dv=%d (need dk == dv in {32,64,128})", fn,
                dk, dv);
  if (chunk_size != 16 && chunk_size != 32 && chunk_size != 64)
    return fail(KDA_ERR_UNSUPPORTED, "%s: chunk_size=%d (need 16, 32 or 64)", fn,
                chunk_size);
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: packed inputs need B == 1", fn);
    if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens needs num_seqs >= 1", fn);
  } else if (num_seqs != 0) {
    return fail(KDA_ERR_INVALID_ARG, "%s: num_seqs=%d without cu_seqlens", fn, num_seqs);
  }
  const int N = cu_seqlens ? num_seqs : B;
  const long long tokens = (long long)B * T;
  if (N == 0) return KDA_OK;
  if (tokens > 0 && (!q || !k || !v || !g || !beta || !o))
    return fail(KDA_ERR_INVALID_ARG, "%s: null input/output pointer", fn);
  const void* ptrs[] = {q, k, v, gmode != kda::kGateLogTok ? g : nullptr, S0, o, S_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is not 16-byte aligned", fn, p);
  if ((beta && !aligned_to(beta, 4)) || (cu_seqlens && !aligned_to(cu_seqlens, 4)) ||
      (g && !aligned_to(g, 4)))
    return fail(KDA_ERR_ALIGNMENT, "%s: beta / cu_seqlens / g not 4-byte aligned", fn);
  if (S_out && o && (const void*)S_out == (const void*)o)
    return fail(KDA_ERR_INVALID_ARG, "%s: o aliases S_out", fn);

  const bool tc_path = use_tensor_core_path(dk, dv, chunk_size, dtype);
  const TcPlan plan = tc_path ? tc_plan(B, T, H, num_seqs) : TcPlan{0, false};
  const int launches = !tc_path ? 1 : plan.fused ? 1 : kda::kTcLaunches;
  cudaEvent_t* ev = t_prof_events;
  if (ev && t_prof_count < launches + 1)
    return fail(KDA_ERR_INVALID_ARG, "%s: %d profiling events, need %d", fn, t_prof_count,
                launches + 1);
  cudaError_t e;
  if (ev && (e = cudaEventRecord(ev[0], stream)) != cudaSuccess) return cuda_fail(e, "event record");
  if (tc_path) {
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, dtype);
    if (need && (!workspace || workspace_bytes < need))
      return fail(KDA_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", fn, workspace_bytes,
                  need);
    if (plan.fused) {
      e = kda::fu::launch_fused(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                static_cast<const __nv_bfloat16*>(v), g, beta, S0,
                                static_cast<__nv_bfloat16*>(o), S_out, cu_seqlens, N, B, T, H, workspace,
                                current_sms(), gmode, stream);
      if (e == cudaSuccess && ev) e = cudaEventRecord(ev[1], stream);
    } else {
      e = kda::launch_chunk_tc(static_cast<const __nv_bfloat16*>(q),
                               static_cast<const __nv_bfloat16*>(k),
                               static_cast<const __nv_bfloat16*>(v), g, beta, S0,
                               static_cast<__nv_bfloat16*>(o), S_out, cu_seqlens, N, B, T, H,
                               max_chunks(B, T, num_seqs, chunk_size), workspace, gmode, plan.seg,
                               t_local_kernel, ev, stream);
    }
  } else if (dtype == KDA_F32) {
    e = dispatch_chunk_simt<float>(dk, chunk_size, q, k, v, g, beta, S0, o, S_out, cu_seqlens, N, T,
                                   H, dv, gmode, stream);
  } else {
    e = dispatch_chunk_simt<__nv_bfloat16>(dk, chunk_size, q, k, v, g, beta, S0, o, S_out,
                                           cu_seqlens, N, T, H, dv, gmode, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (ev && launches == 1 && (e = cudaEventRecord(ev[1], stream)) != cudaSuccess)
    return cuda_fail(e, "event record");
  return KDA_OK;
}

kda_status_t recurrent_step_impl(const char* fn, const void* q, const void* k, const void* v,
                                const void* g, const float* beta, float* S, void* o, int N, int H,
                                int dk, int dv, kda_dtype_t dtype, int gmode, cudaStream_t stream) {
  t_err[0] = 0;
  if (N < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes N=%d H=%d", fn, N, H);
  if (dtype != KDA_BF16 && dtype != KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dtype);
  if (!supported_head(dk, dv))
    return fail(KDA_ERR_UNSUPPORTED,
                "%s: dk=%d dv=%d (need dk == dv in {32,64,128})", fn, dk, dv);
  if (N == 0) return KDA_OK;
  if (!q || !k || !v || !g || !beta || !S || !o)
    return fail(KDA_ERR_INVALID_ARG, "%s: null pointer", fn);
  const unsigned esz = dtype == KDA_F32 ? 4u : 2u;
  if (!aligned16(S)) return fail(KDA_ERR_ALIGNMENT, "%s: S %p is not 16-byte aligned", fn, (const void*)S);
  const void* elem[] = {q, k, v, o};
  for (const void* p : elem)
    if (!aligned_to(p, esz)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is misaligned", fn, p);
  if (!aligned_to(g, gmode == kda::kGateLogitBf16 ? 2 : 4) || !aligned_to(beta, 4))
    return fail(KDA_ERR_ALIGNMENT, "%s: g / beta not element-aligned", fn);
  cudaError_t e = dtype == KDA_F32
                      ? dispatch_decode<float>(dk, q, k, v, g, beta, S, o, N, H, gmode, stream)
                      : dispatch_decode<__nv_bfloat16>(dk, q, k, v, g, beta, S, o, N, H, gmode, stream);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return KDA_OK;
}

}  // namespace

extern "C" {

const char* kda_last_error(void) { return t_err; }

int kda_version(void) { return 100; }

int kda_chunk_fwd_launches(int dk, int dv, int chunk_size, kda_dtype_t dtype) {
  return use_tensor_core_path(dk, dv, chunk_size, dtype) ? kda::kTcLaunches : 1;
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs) {
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || !supported_head(dk, dv)) return 0;
  return kda::bwd::bwd_workspace_bytes(B, T, H, dk, num_seqs);
}

// The backward of both gate layouts: gate = kGateLogCh (g, dg [.., H, dk]) or
// kGateLogTok (g, dg [.., H]).
static kda_status_t chunk_bwd_impl(const char* fn, int gate, const void* q, const void* k, const void* v,
                                   const float* g, const float* beta, const float* S0, const void* dout,
                                   const float* dS_T, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                                   float* dS0, const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                                   int dkh, int dvh, kda_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  t_err[0] = 0;
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0)
    return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d num_seqs=%d", fn, B, T, H, num_seqs);
  if (dtype != KDA_BF16 && dtype != KDA_F32) return fail(KDA_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dtype);
  if (!supported_head(dkh, dvh))
    return fail(KDA_ERR_UNSUPPORTED, "%s: dk=%d dv=%d (need dk == dv in {32,64,128})", fn, dkh, dvh);
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: packed inputs need B == 1", fn);
    if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens needs num_seqs >= 1", fn);
  } else if (num_seqs != 0) {
    return fail(KDA_ERR_INVALID_ARG, "%s: num_seqs=%d without cu_seqlens", fn, num_seqs);
  }
  const int N = cu_seqlens ? num_seqs : B;
  if (N == 0) return KDA_OK;
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta))
    return fail(KDA_ERR_INVALID_ARG, "%s: null input/output pointer", fn);
  const unsigned esz = dtype == KDA_F32 ? 4u : 2u;
  const void* in_ptrs[] = {q, k, v, dout};
  for (const void* p : in_ptrs)
    if (p && !aligned_to(p, esz)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is misaligned", fn, p);
  const void* f_ptrs[] = {g, beta, S0, dS_T, dq, dk, dv, dg, dbeta, dS0, cu_seqlens, workspace};
  for (const void* p : f_ptrs)
    if (p && !aligned_to(p, 4)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is not 4-byte aligned", fn, p);
  {  // outputs are written while inputs are still read (in reverse chunk order): no aliasing
    const void* outs[] = {dq, dk, dv, dg, dbeta, dS0, workspace};
    const void* ins[] = {q, k, v, g, beta, S0, dout, dS_T};
    for (int i = 0; i < 7; ++i) {
      if (!outs[i]) continue;
      for (const void* p : ins)
        if (p == outs[i]) return fail(KDA_ERR_INVALID_ARG, "%s: an output aliases an input (%p)", fn, p);
      for (int j = i + 1; j < 7; ++j)
        if (outs[j] == outs[i]) return fail(KDA_ERR_INVALID_ARG, "%s: two outputs alias (%p)", fn, outs[i]);
    }
  }
  const size_t need = kda_chunk_bwd_workspace_size(B, T, H, dkh, dvh, num_seqs);
  if (need && (!workspace || workspace_bytes < need))
    return fail(KDA_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", fn, workspace_bytes, need);
  float* ck = static_cast<float*>(workspace);
  cudaError_t e = cudaErrorInvalidValue;
#define KDA_BWD_CASE(TT, DD)                                                                            \
  e = gate == kda::kGateLogTok                                                                           \
          ? kda::bwd::launch_chunk_bwd<TT, DD, kda::kGateLogTok>(q, k, v, g, beta, S0, dout, dS_T, dq, dk, \
                                                                 dv, dg, dbeta, dS0, cu_seqlens, N, T, H,  \
                                                                 ck, stream)                               \
          : kda::bwd::launch_chunk_bwd<TT, DD, kda::kGateLogCh>(q, k, v, g, beta, S0, dout, dS_T, dq, dk,  \
                                                                dv, dg, dbeta, dS0, cu_seqlens, N, T, H,   \
                                                                ck, stream)
  if (dtype == KDA_F32) {
    if (dkh == 32) KDA_BWD_CASE(float, 32); else if (dkh == 64) KDA_BWD_CASE(float, 64); else KDA_BWD_CASE(float, 128);
  } else {
    if (dkh == 32) KDA_BWD_CASE(__nv_bfloat16, 32);
    else if (dkh == 64) KDA_BWD_CASE(__nv_bfloat16, 64);
    else KDA_BWD_CASE(__nv_bfloat16, 128);
  }
#undef KDA_BWD_CASE
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return KDA_OK;
}

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, const void* dout, const float* dS_T, float* dq, float* dk,
                           float* dv, float* dg, float* dbeta, float* dS0, const int32_t* cu_seqlens,
                           int num_seqs, int B, int T, int H, int dkh, int dvh, kda_dtype_t dtype,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return chunk_bwd_impl("kda_chunk_bwd", kda::kGateLogCh, q, k, v, g, beta, S0, dout, dS_T, dq, dk, dv, dg,
                        dbeta, dS0, cu_seqlens, num_seqs, B, T, H, dkh, dvh, dtype, workspace, workspace_bytes,
                        stream);
}

kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                               const float* S0, const void* dout, const float* dS_T, float* dq, float* dk,
                               float* dv, float* dg, float* dbeta, float* dS0, const int32_t* cu_seqlens,
                               int num_seqs, int B, int T, int H, int dkh, int dvh, kda_dtype_t dtype,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return chunk_bwd_impl("kda_gdn_chunk_bwd", kda::kGateLogTok, q, k, v, g, beta, S0, dout, dS_T, dq, dk, dv, dg,
                        dbeta, dS0, cu_seqlens, num_seqs, B, T, H, dkh, dvh, dtype, workspace, workspace_bytes,
                        stream);
}

size_t kda_chunk_bwd_prep_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs) {
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || !supported_head(dk, dv)) return 0;
  const size_t ck = kda::bwd::bwd_workspace_bytes(B, T, H, dk, num_seqs);
  return kda::bwd::prep_bwd_layout(ck, (long long)B * T * H, dk).total;
}

kda_status_t kda_chunk_bwd_prep(const void* q, const void* k, const void* v, const void* a, kda_dtype_t a_dtype,
                                const float* b, const float* S0, const void* dout, const float* dS_T, float* dq,
                                float* dk, float* dv, float* da, float* db, float* dS0, const int32_t* cu_seqlens,
                                int num_seqs, int B, int T, int H, int dkh, int dvh, kda_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const char* fn = "kda_chunk_bwd_prep";
  t_err[0] = 0;
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0)
    return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d num_seqs=%d", fn, B, T, H, num_seqs);
  if (dtype != KDA_BF16 && dtype != KDA_F32) return fail(KDA_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dtype);
  if (a_dtype != KDA_BF16 && a_dtype != KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "%s: unknown a_dtype %d", fn, (int)a_dtype);
  if (!supported_head(dkh, dvh))
    return fail(KDA_ERR_UNSUPPORTED, "%s: dk=%d dv=%d (need dk == dv in {32,64,128})", fn, dkh, dvh);
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: packed inputs need B == 1", fn);
    if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens needs num_seqs >= 1", fn);
  } else if (num_seqs != 0) {
    return fail(KDA_ERR_INVALID_ARG, "%s: num_seqs=%d without cu_seqlens", fn, num_seqs);
  }
  const int N = cu_seqlens ? num_seqs : B;
  if (N == 0) return KDA_OK;
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !a || !b || !dout || !dq || !dk || !dv || !da || !db))
    return fail(KDA_ERR_INVALID_ARG, "%s: null input/output pointer", fn);
  const unsigned esz = dtype == KDA_F32 ? 4u : 2u, aesz = a_dtype == KDA_F32 ? 4u : 2u;
  const void* in_ptrs[] = {q, k, v, dout};
  for (const void* p : in_ptrs)
    if (p && !aligned_to(p, esz)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is misaligned", fn, p);
  if (a && !aligned_to(a, aesz)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is misaligned", fn, a);
  const void* f_ptrs[] = {b, S0, dS_T, dq, dk, dv, da, db, dS0, cu_seqlens, workspace};
  for (const void* p : f_ptrs)
    if (p && !aligned_to(p, 4)) return fail(KDA_ERR_ALIGNMENT, "%s: pointer %p is not 4-byte aligned", fn, p);
  {  // outputs are written while inputs are still read: no aliasing
    const void* outs[] = {dq, dk, dv, da, db, dS0, workspace};
    const void* ins[] = {q, k, v, a, b, S0, dout, dS_T};
    for (int i = 0; i < 7; ++i) {
      if (!outs[i]) continue;
      for (const void* p : ins)
        if (p == outs[i]) return fail(KDA_ERR_INVALID_ARG, "%s: an output aliases an input (%p)", fn, p);
      for (int j = i + 1; j < 7; ++j)
        if (outs[j] == outs[i]) return fail(KDA_ERR_INVALID_ARG, "%s: two outputs alias (%p)", fn, outs[i]);
    }
  }
  const size_t need = kda_chunk_bwd_prep_workspace_size(B, T, H, dkh, dvh, num_seqs);
  if (need && (!workspace || workspace_bytes < need))
    return fail(KDA_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", fn, workspace_bytes, need);
  const size_t ck = kda::bwd::bwd_workspace_bytes(B, T, H, dkh, num_seqs);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int a_bf16 = a_dtype == KDA_BF16;
  cudaError_t e = cudaErrorInvalidValue;
#define KDA_BWD_PREP_CASE(TT, DD)                                                                           \
  e = kda::bwd::launch_chunk_bwd_prep<TT, DD>(q, k, v, a, a_bf16, b, S0, dout, dS_T, dq, dk, dv, da, db, dS0, \
                                              cu_seqlens, N, B, T, H, ck, ws, stream)
  if (dtype == KDA_F32) {
    if (dkh == 32) KDA_BWD_PREP_CASE(float, 32); else if (dkh == 64) KDA_BWD_PREP_CASE(float, 64); else KDA_BWD_PREP_CASE(float, 128);
  } else {
    if (dkh == 32) KDA_BWD_PREP_CASE(__nv_bfloat16, 32);
    else if (dkh == 64) KDA_BWD_PREP_CASE(__nv_bfloat16, 64);
    else KDA_BWD_PREP_CASE(__nv_bfloat16, 128);
  }
#undef KDA_BWD_PREP_CASE
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return KDA_OK;
}

kda_status_t kda_set_segment_chunks(int chunks) {
  t_err[0] = 0;
  t_seg_force = chunks;
  return KDA_OK;
}

int kda_segment_chunks(int B, int T, int H, int num_seqs) {
  return tc_plan(B, T, H, num_seqs).seg;
}

kda_status_t kda_set_prefill_path(int path) {
  t_err[0] = 0;
  if (path != kda::kPathAuto && path != kda::kPathFused && path != kda::kPathTwoKernel)
    return fail(KDA_ERR_INVALID_ARG, "kda_set_prefill_path: path %d", path);
  t_prefill_path = path;
  return KDA_OK;
}

int kda_chunk_fwd_phases(int B, int T, int H, int num_seqs, int dk, int dv, int chunk_size, kda_dtype_t dtype) {
  if (!use_tensor_core_path(dk, dv, chunk_size, dtype)) return 1;
  return tc_plan(B, T, H, num_seqs).fused ? 1 : kda::kTcLaunches;
}

kda_status_t kda_set_local_kernel(int variant) {
  t_err[0] = 0;
  if (variant != 0 && variant != 1) return fail(KDA_ERR_INVALID_ARG, "kda_set_local_kernel: variant %d", variant);
  t_local_kernel = variant;
  return KDA_OK;
}

kda_status_t kda_profile_events(cudaEvent_t* events, int count) {
  t_err[0] = 0;
  if (events && count <= 0) return fail(KDA_ERR_INVALID_ARG, "kda_profile_events: count=%d", count);
  t_prof_events = events;
  t_prof_count = events ? count : 0;
  return KDA_OK;
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                    int chunk_size, kda_dtype_t dtype) {
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || chunk_size <= 0) return 0;
  if (!use_tensor_core_path(dk, dv, chunk_size, dtype)) return 0;
  const int N = num_seqs > 0 ? num_seqs : B;
  const TcPlan plan = tc_plan(B, T, H, num_seqs);
  if (plan.fused) return kda::fu::fused_workspace_bytes(num_seqs, (long long)N * H);
  return kda::tc_workspace_layout(max_chunks(B, T, num_seqs, chunk_size), H, (long long)N * H, T, plan.seg,
                                  num_seqs).total;
}

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, void* o, float* S_out,
                           const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                           int dk, int dv, int chunk_size, kda_dtype_t dtype,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return chunk_fwd_impl("kda_chunk_fwd", q, k, v, g, beta, S0, o, S_out, cu_seqlens, num_seqs, B, T,
                        H, dk, dv, chunk_size, dtype, workspace, workspace_bytes, kda::kGateLogCh, stream);
}

kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* S0, void* o, float* S_out,
                               const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                               int dk, int dv, int chunk_size, kda_dtype_t dtype,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return chunk_fwd_impl("kda_gdn_chunk_fwd", q, k, v, g, beta, S0, o, S_out, cu_seqlens, num_seqs,
                        B, T, H, dk, dv, chunk_size, dtype, workspace, workspace_bytes, kda::kGateLogTok,
                        stream);
}

kda_status_t kda_chunk_fwd_prep(const void* q, const void* k, const void* v, const void* a,
                                kda_dtype_t a_dtype, const float* b, const float* S0, void* o,
                                float* S_out, const int32_t* cu_seqlens, int num_seqs, int B, int T,
                                int H, int dk, int dv, int chunk_size, kda_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (a_dtype != KDA_BF16 && a_dtype != KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_prep: unknown a_dtype %d", (int)a_dtype);
  return chunk_fwd_impl("kda_chunk_fwd_prep", q, k, v, a, b, S0, o, S_out, cu_seqlens, num_seqs, B, T,
                        H, dk, dv, chunk_size, dtype, workspace, workspace_bytes,
                        a_dtype == KDA_BF16 ? kda::kGateLogitBf16 : kda::kGateLogitF32, stream);
}

kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* S, void* o, int N, int H, int dk,
                                int dv, kda_dtype_t dtype, cudaStream_t stream) {
  return recurrent_step_impl("kda_recurrent_step", q, k, v, g, beta, S, o, N, H, dk, dv, dtype,
                             kda::kGateLogCh, stream);
}

kda_status_t kda_gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, float* S, void* o, int N, int H, int dk,
                                    int dv, kda_dtype_t dtype, cudaStream_t stream) {
  return recurrent_step_impl("kda_gdn_recurrent_step", q, k, v, g, beta, S, o, N, H, dk, dv, dtype,
                             kda::kGateLogTok, stream);
}

kda_status_t kda_recurrent_step_prep(const void* q, const void* k, const void* v, const void* a,
                                     kda_dtype_t a_dtype, const float* b, float* S, void* o, int N,
                                     int H, int dk, int dv, kda_dtype_t dtype, cudaStream_t stream) {
  if (a_dtype != KDA_BF16 && a_dtype != KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "kda_recurrent_step_prep: unknown a_dtype %d", (int)a_dtype);
  return recurrent_step_impl("kda_recurrent_step_prep", q, k, v, a, b, S, o, N, H, dk, dv, dtype,
                             a_dtype == KDA_BF16 ? kda::kGateLogitBf16 : kda::kGateLogitF32, stream);
}

// ---------------------------------------------------------------------------
// Prefill from host buffers.
// ---------------------------------------------------------------------------
namespace {
// Rows of one pipeline group and the device workspace a group needs (the
// largest over the group sizes that occur: a smaller group may take another
// path).
struct HostPlan {
  int pieces, rows, last_rows;
  size_t ws;
};
HostPlan host_plan(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size, kda_dtype_t dtype,
                   int pieces) {
  HostPlan p;
  p.pieces = num_seqs > 0 || B <= 1 ? 1 : std::max(1, std::min(pieces, B));
  p.rows = num_seqs > 0 ? B : (B + p.pieces - 1) / p.pieces;
  p.pieces = num_seqs > 0 ? 1 : (B + p.rows - 1) / std::max(p.rows, 1);
  p.last_rows = B - (p.pieces - 1) * p.rows;
  p.ws = std::max(kda_chunk_fwd_workspace_size(p.rows, T, H, dk, dv, num_seqs, chunk_size, dtype),
                  kda_chunk_fwd_workspace_size(p.last_rows, T, H, dk, dv, num_seqs, chunk_size, dtype));
  return p;
}
}  // namespace

size_t kda_chunk_fwd_host_buffer_size(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size,
                                      kda_dtype_t dtype, int pieces) {
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || pieces < 1 || !supported_head(dk, dv)) return 0;
  if (dtype != KDA_BF16 && dtype != KDA_F32) return 0;
  const int N = num_seqs > 0 ? num_seqs : B;
  const HostPlan plan = host_plan(B, T, H, dk, dv, num_seqs, chunk_size, dtype, pieces);
  const size_t esz = dtype == KDA_F32 ? 4 : 2;
  return kda::host::host_layout(kda::host::host_sizes(B, T, H, dk, dv, N, num_seqs, esz), plan.ws).total;
}

kda_status_t kda_chunk_fwd_host(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* S0, void* o, float* S_out,
                                const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                                int dv, int chunk_size, kda_dtype_t dtype, int pieces,
                                void* device_buffer, size_t device_buffer_bytes, cudaStream_t compute,
                                cudaStream_t copy_in, cudaStream_t copy_out) {
  const char* fn = "kda_chunk_fwd_host";
  t_err[0] = 0;
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || pieces < 1)
    return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d num_seqs=%d pieces=%d", fn, B, T, H,
                num_seqs, pieces);
  if (dtype != KDA_BF16 && dtype != KDA_F32) return fail(KDA_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dtype);
  if (!supported_head(dk, dv))
    return fail(KDA_ERR_UNSUPPORTED, "%s: dk=%d dv=%d (need dk == dv in {32,64,128})", fn, dk, dv);
  if (cu_seqlens ? (B != 1 || num_seqs < 1) : num_seqs != 0)
    return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens needs B == 1 and num_seqs >= 1 (num_seqs=0 without)", fn);
  const int N = cu_seqlens ? num_seqs : B;
  if (N == 0) return KDA_OK;
  const long long tokens = (long long)B * T;
  if (tokens > 0 && (!q || !k || !v || !g || !beta || !o))
    return fail(KDA_ERR_INVALID_ARG, "%s: null host input/output pointer", fn);
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) & (kda::host::kAlign - 1)))
    return fail(KDA_ERR_ALIGNMENT, "%s: device_buffer must be a %zu-byte aligned device pointer", fn,
                kda::host::kAlign);
  const HostPlan plan = host_plan(B, T, H, dk, dv, num_seqs, chunk_size, dtype, pieces);
  const size_t esz = dtype == KDA_F32 ? 4 : 2;
  const kda::host::HostSizes sz = kda::host::host_sizes(B, T, H, dk, dv, N, num_seqs, esz);
  const kda::host::HostLayout L = kda::host::host_layout(sz, plan.ws);
  if (device_buffer_bytes < L.total)
    return fail(KDA_ERR_WORKSPACE, "%s: device_buffer %zu bytes, need %zu (kda_chunk_fwd_host_buffer_size)", fn,
                device_buffer_bytes, L.total);
  kda::host::HostEvents* ev = nullptr;
  cudaError_t e = kda::host::host_events(&ev);
  if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_host: events");
  uint8_t* base = static_cast<uint8_t*>(device_buffer);
  // the inner prefill calls record no profiling events of the caller's
  cudaEvent_t* saved_ev = t_prof_events;
  const int saved_cnt = t_prof_count;
  t_prof_events = nullptr;
  t_prof_count = 0;
  kda_status_t st = KDA_OK;
  auto h2d = [&](size_t off, const void* src, size_t bytes) {
    if (e == cudaSuccess && bytes) e = cudaMemcpyAsync(base + off, src, bytes, cudaMemcpyHostToDevice, copy_in);
  };
  auto d2h = [&](void* dst, size_t off, size_t bytes) {
    if (e == cudaSuccess && bytes) e = cudaMemcpyAsync(dst, base + off, bytes, cudaMemcpyDeviceToHost, copy_out);
  };
  auto cu8 = [](const void* p) { return static_cast<const uint8_t*>(p); };
  // earlier work on `compute` (which may still use the buffer) comes first
  if ((e = cudaEventRecord(ev->done, compute)) == cudaSuccess) e = cudaStreamWaitEvent(copy_in, ev->done, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(copy_out, ev->done, 0);
  h2d(L.cu, cu_seqlens, sz.cu);
  // per-row strides of every tensor (rows = batch rows; packed: one row)
  const size_t row_q = sz.q / std::max(B, 1), row_v = sz.v / std::max(B, 1), row_g = sz.g / std::max(B, 1);
  const size_t row_b = sz.beta / std::max(B, 1), row_s = sz.state / N;
  for (int p = 0; p < plan.pieces && e == cudaSuccess && st == KDA_OK; ++p) {
    const int b0 = p * plan.rows, nb = std::min(plan.rows, B - b0);
    // states: packed inputs have N = num_seqs state rows, all in the one group
    const int s0r = cu_seqlens ? 0 : b0, ns = cu_seqlens ? N : nb;
    h2d(L.q + b0 * row_q, cu8(q) + b0 * row_q, nb * row_q);
    h2d(L.k + b0 * row_q, cu8(k) + b0 * row_q, nb * row_q);
    h2d(L.v + b0 * row_v, cu8(v) + b0 * row_v, nb * row_v);
    h2d(L.g + b0 * row_g, cu8(g) + b0 * row_g, nb * row_g);
    h2d(L.beta + b0 * row_b, cu8(beta) + b0 * row_b, nb * row_b);
    if (S0) h2d(L.S0 + s0r * row_s, cu8(S0) + s0r * row_s, ns * row_s);
    if (e == cudaSuccess) e = cudaEventRecord(ev->in, copy_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(compute, ev->in, 0);
    if (e != cudaSuccess) break;
    st = kda_chunk_fwd(base + L.q + b0 * row_q, base + L.k + b0 * row_q, base + L.v + b0 * row_v,
                       reinterpret_cast<const float*>(base + L.g + b0 * row_g),
                       reinterpret_cast<const float*>(base + L.beta + b0 * row_b),
                       S0 ? reinterpret_cast<const float*>(base + L.S0 + s0r * row_s) : nullptr,
                       base + L.o + b0 * row_v,
                       S_out ? reinterpret_cast<float*>(base + L.S_out + s0r * row_s) : nullptr,
                       cu_seqlens ? reinterpret_cast<const int32_t*>(base + L.cu) : nullptr, num_seqs, nb, T, H,
                       dk, dv, chunk_size, dtype, plan.ws ? base + L.ws : nullptr, plan.ws, compute);
    if (st != KDA_OK) break;
    if ((e = cudaEventRecord(ev->done, compute)) == cudaSuccess) e = cudaStreamWaitEvent(copy_out, ev->done, 0);
    d2h(static_cast<uint8_t*>(o) + b0 * row_v, L.o + b0 * row_v, nb * row_v);
    if (S_out) d2h(reinterpret_cast<uint8_t*>(S_out) + s0r * row_s, L.S_out + s0r * row_s, ns * row_s);
  }
  // the caller synchronises `compute` to see everything, the copies back included
  if (e == cudaSuccess && st == KDA_OK && (e = cudaEventRecord(ev->out, copy_out)) == cudaSuccess)
    e = cudaStreamWaitEvent(compute, ev->out, 0);
  t_prof_events = saved_ev;
  t_prof_count = saved_cnt;
  if (st != KDA_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return KDA_OK;
}

// ---------------------------------------------------------------------------
// Prefill without any caller-provided workspace.
//
// Some callers cannot allocate device memory: a plug-in that receives only
// input and output pointers from a host framework that owns the whole device
// memory pool, or code that must not call cudaMalloc because it implicitly
// synchronises the device.  For them the scratch the tensor-core prefill
// needs (its per-chunk operand images) lives in this file-scope device array
// instead.  Every GPU that loads the library keeps it until process exit.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mutex;
// Device address of g_noalloc_scratch, per device ordinal, with the context
// that was current when it was looked up: the address belongs to the module
// instance of that context, so a different context on the same ordinal (a
// non-primary context, or the primary one re-created after cudaDeviceReset)
// looks it up again.
struct NoallocEntry {
  void* ctx;
  void* ptr;
};
NoallocEntry g_noalloc[256] = {};

// cuCtxGetCurrent, fetched once from the driver through the runtime (no link
// against the driver library).
typedef int (*CtxGetCurrentFn)(void**);
CtxGetCurrentFn ctx_get_current() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Host code only ever sees a host-side stand-in for g_noalloc_scratch, so the
// real device address is looked up with the device current, once per device
// and context.
kda_status_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 256) return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_noalloc: device %d", dev);
  void* ctx = nullptr;
  const CtxGetCurrentFn get = ctx_get_current();
  if (!get) return fail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: cuCtxGetCurrent unavailable");
  if (get(&ctx) != 0 || !ctx) {
    // No context current on this thread yet: cudaSetDevice (CUDA 12+) makes the
    // device's primary context current (the device itself does not change).  A
    // context the caller made current is never replaced.
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaSetDevice");
    if (get(&ctx) != 0 || !ctx) return fail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: no current CUDA context");
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoallocEntry& ent = g_noalloc[dev];
  if (!ent.ptr || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "kda_chunk_fwd_noalloc: cudaGetSymbolAddress");
    ent.ctx = ctx;
    ent.ptr = p;
  }
  *out = ent.ptr;
  return KDA_OK;
}
}  // namespace

kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* S0, void* o, float* S_out,
                                   const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                                   int dk, int dv, int chunk_size, kda_dtype_t dtype,
                                   cudaStream_t stream) {
  t_err[0] = 0;
  if (B < 0 || T < 0 || H <= 0 || num_seqs < 0 || chunk_size <= 0)
    return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: bad sizes B=%d T=%d H=%d num_seqs=%d", B, T,
                H, num_seqs);
  size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, dtype);
  // The automatic sequence segments are a speed choice whose state maps take
  // scratch too: where they would not fit, this call runs without them.
  const int seg_setting = t_seg_force;
  if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES && seg_setting == 0) {
    t_seg_force = -1;
    need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, dtype);
  }
  if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) {
    t_seg_force = seg_setting;
    return fail(KDA_ERR_WORKSPACE,
                "kda_chunk_fwd_noalloc: these sizes need %zu bytes of scratch, more than the built-in "
                "%zu-byte array; use kda_chunk_fwd with a caller-provided workspace",
                need, (size_t)KDA_NOALLOC_SCRATCH_BYTES);
  }
  void* scratch = nullptr;
  if (need > 0) {
    const kda_status_t st = noalloc_scratch(&scratch);
    if (st != KDA_OK) {
      t_seg_force = seg_setting;
      return st;
    }
  }
  const kda_status_t st = kda_chunk_fwd(q, k, v, g, beta, S0, o, S_out, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                        chunk_size, dtype, scratch, need, stream);
  t_seg_force = seg_setting;
  return st;
}

}  // extern "C"

namespace kda {
// One thread waits, with the kernels' own bounded wait, on an mbarrier that
// nothing ever arrives at; the wait gives up after limit_ns and raises the
// device error word.
__global__ void kda_bounded_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
    (void)ptx::mbar_wait_bounded(&bar, 0, limit_ns);
  }
}
}  // namespace kda

extern "C" {

kda_status_t kda_selftest_bounded_wait(unsigned long long limit_ns, cudaStream_t stream) {
  t_err[0] = 0;
  if (limit_ns == 0 || limit_ns > 1000000000ull)
    return fail(KDA_ERR_INVALID_ARG, "kda_selftest_bounded_wait: limit_ns=%llu (need 1 .. 1e9)", limit_ns);
  kda::kda_bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_bounded_wait launch");
  return KDA_OK;
}

kda_status_t kda_device_error(int* code, cudaStream_t stream) {
  t_err[0] = 0;
  if (!code) return fail(KDA_ERR_INVALID_ARG, "kda_device_error: null code");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_device_error: synchronize");
  int h = 0;
  e = cudaMemcpyFromSymbol(&h, kda::g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "kda_device_error: read");
  const int zero = 0;
  e = cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "kda_device_error: clear");
  *code = h;
  return KDA_OK;
}

}  // extern "C"
