// kda_common.cuh -- small device helpers shared by the KDA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace kda {

// Host-side, per-device one-time setup (kernel attributes), safe to call from
// several host threads at once: `setup` runs once per device and object.
constexpr int kMaxDevices = 64;
struct PerDeviceOnce {
  std::mutex mu;
  bool done[kMaxDevices] = {};
};
template <typename F>
inline cudaError_t run_once_per_device(PerDeviceOnce& once, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return setup();
  std::lock_guard<std::mutex> lock(once.mu);
  if (once.done[dev]) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess) once.done[dev] = true;
  return e;
}
// SM count of the current device (cached per device, thread-safe).
inline int current_sm_count() {
  static std::mutex mu;
  static int sms[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= kMaxDevices) {
    int n = 0;
    return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms[dev] = 0;
  return sms[dev];
}

// Device-side error word.  Bounded waits set it (never trap) when they give
// up; the host reads and clears it through kda_device_error().
__device__ int g_device_error;

// Codes match kda_status_t: a malformed cu_seqlens table seen on the device
// (KDA_ERR_INVALID_ARG), a bounded wait that gave up (KDA_ERR_DEVICE_TIMEOUT).
enum : int { kDevErrNone = 0, kDevErrBadSeqlens = 1, kDevErrWaitTimeout = 6 };

__device__ __forceinline__ void raise_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

// Token range [t0, t1) of packed sequence n, checked: a sequence whose range
// is not inside [0, total] with t0 <= t1 raises the device error word and is
// treated as empty (the caller then reads and writes nothing for it).
__device__ __forceinline__ bool checked_seq_range(const int32_t* cu, int n, long long total, long long* t0,
                                                  long long* t1) {
  const long long a = cu[n], b = cu[n + 1];
  if (a < 0 || b < a || b > total) {
    raise_device_error(kDevErrBadSeqlens);
    *t0 = *t1 = 0;
    return false;
  }
  *t0 = a;
  *t1 = b;
  return true;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Division of n < 2^31 by a fixed divisor d >= 1 with one multiply-high
// ("division by invariant integers using multiplication", Granlund and
// Montgomery, 1994): l = ceil(log2 d), m = ceil(2^(32+l) / d) - 2^32 (fits in
// 32 bits), q = (umulhi(n, m) + n) >> l; n + umulhi(n, m) < 2^32 for n < 2^31.
struct FastDiv {
  uint32_t d, mul;
  int shift;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0};
  while ((1ull << f.shift) < d) ++f.shift;
  const unsigned long long two32 = 1ull << 32;
  // ceil(2^(32+l) / d) - 2^32 = floor((2^(32+l) - 1) / d) + 1 - 2^32
  const unsigned long long num = (two32 << f.shift) - 1ull;  // < 2^63 for l <= 31
  f.mul = (uint32_t)(num / d + 1ull - two32);
  return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shift;
}

// What the gate argument holds and how it is laid out.
enum GateMode : int {
  kGateLogCh = 0,      // log alpha, fp32 [.., H, dk]: one decay per key channel (KDA)
  kGateLogTok = 1,     // log alpha, fp32 [.., H]: one decay per token and head (Gated DeltaNet)
  kGateLogitF32 = 2,   // raw logit a, fp32 [.., H, dk]; log alpha = -softplus(a), and the
                       // call also L2-normalises q, k and takes beta = sigmoid(b)
  kGateLogitBf16 = 3,  // the same with a in bf16
};
__host__ __device__ constexpr bool gate_prep(int m) { return m >= kGateLogitF32; }

// -softplus(a) = -(max(a, 0) + log(1 + e^{-|a|})), finite for every finite a.
__device__ __forceinline__ float neg_softplus(float a) {
  return -(fmaxf(a, 0.f) + log1pf(__expf(-fabsf(a))));
}
__device__ __forceinline__ float sigmoid_f(float b) { return 1.f / (1.f + __expf(-b)); }

// log alpha of key channel c of token-head row `row` (row = token * H + head).
__device__ __forceinline__ float gate_log(const void* gate, int mode, size_t row, int DK, int c) {
  switch (mode) {
    case kGateLogCh: return static_cast<const float*>(gate)[row * DK + c];
    case kGateLogTok: return static_cast<const float*>(gate)[row];
    case kGateLogitF32: return neg_softplus(static_cast<const float*>(gate)[row * DK + c]);
    default: return neg_softplus(__bfloat162float(static_cast<const __nv_bfloat16*>(gate)[row * DK + c]));
  }
}
// beta of token-head row `row`: given, or sigmoid of the given logit.
__device__ __forceinline__ float beta_of(const float* beta, int mode, size_t row) {
  return gate_prep(mode) ? sigmoid_f(beta[row]) : beta[row];
}

__device__ __forceinline__ float4 f4_scale(float4 a, float s) {
  return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
__device__ __forceinline__ float4 f4_fma(float s, float4 a, float4 acc) {
  return make_float4(fmaf(s, a.x, acc.x), fmaf(s, a.y, acc.y), fmaf(s, a.z, acc.z),
                     fmaf(s, a.w, acc.w));
}

}  // namespace kda
