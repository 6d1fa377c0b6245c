// kda_host.cuh -- the prefill from HOST buffers (kda_chunk_fwd_host): copies
// the inputs to the device, runs kda_chunk_fwd and copies o and S_out back,
// pipelined over groups of batch rows on three caller streams, so that the
// host->device copy of group p+1, the prefill of group p and the device->host
// copy of group p-1 run at the same time (both copy directions and the SMs).
//
// Device memory: one caller-provided buffer, carved here into the device
// copies of every tensor and the prefill's workspace for one group of rows.
#pragma once
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "kda_common.cuh"

namespace kda {
namespace host {

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Byte sizes of the tensors of one call.
struct HostSizes {
  size_t q, v, g, beta, state, cu;
};
inline HostSizes host_sizes(int B, int T, int H, int dk, int dv, int N, int num_seqs, size_t esz) {
  const size_t rows = (size_t)B * (size_t)T * (size_t)H;
  HostSizes s;
  s.q = rows * dk * esz;
  s.v = rows * dv * esz;
  s.g = rows * dk * sizeof(float);
  s.beta = rows * sizeof(float);
  s.state = (size_t)N * H * dk * dv * sizeof(float);
  s.cu = num_seqs > 0 ? (size_t)(num_seqs + 1) * sizeof(int32_t) : 0;
  return s;
}

// Offsets of the device copies inside the caller's buffer: q, k, v, g, beta,
// S0, o, S_out, cu_seqlens, then the workspace.
struct HostLayout {
  size_t q, k, v, g, beta, S0, o, S_out, cu, ws, total;
};
inline HostLayout host_layout(const HostSizes& s, size_t ws_bytes) {
  HostLayout L;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at = round_up(at + bytes);
    return here;
  };
  L.q = take(s.q);
  L.k = take(s.q);
  L.v = take(s.v);
  L.g = take(s.g);
  L.beta = take(s.beta);
  L.S0 = take(s.state);
  L.o = take(s.v);
  L.S_out = take(s.state);
  L.cu = take(s.cu);
  L.ws = take(ws_bytes);
  L.total = at;
  return L;
}

// Three events per (host thread, device), created on first use and reused:
// a stream waits on an event's record as it stood when the wait was enqueued,
// so each event can be recorded again right after the wait that reads it.
struct HostEvents {
  cudaEvent_t in = nullptr, done = nullptr, out = nullptr;
};
inline cudaError_t host_events(HostEvents** out) {
  thread_local HostEvents ev[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  HostEvents& h = ev[dev];
  cudaEvent_t* all[3] = {&h.in, &h.done, &h.out};
  for (cudaEvent_t* p : all)
    if (!*p && (e = cudaEventCreateWithFlags(p, cudaEventDisableTiming)) != cudaSuccess) return e;
  *out = &h;
  return cudaSuccess;
}

}  // namespace host
}  // namespace kda
