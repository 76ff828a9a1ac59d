// wkv_forward_host (declared in include/wkv.h): the sequence forward over
// host-resident k, v and out. The sequence is cut into segments of whole
// tokens; segment s is copied to the device on one library stream, computed
// by wkv_forward on the caller's stream from the state after segment s-1, and
// its outputs copied back on a second library stream. Two segments are in
// flight (double-buffered device copies), so the host-to-device copy of
// segment s+1, the compute of segment s and the device-to-host copy of
// segment s-1 run side by side. Host code only: it calls the public
// wkv_forward and the CUDA runtime's copies and events.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/wkv.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kDefaultSegBytes = 64ll << 20;  // k and v of one segment, by default

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The copy streams and the events that order them against the caller's
// stream, per device; created on first use. mu serialises the queueing of one
// call's work (the events are shared).
struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t s_in = nullptr, s_in2 = nullptr, s_out = nullptr;  // k in, v in, out back
  cudaEvent_t fork = nullptr;
  cudaEvent_t loaded[2] = {}, loaded2[2] = {}, computed[2] = {}, unloaded[2] = {};
};
HostPipe g_pipe[kMaxDevices];

bool pipe_ready(HostPipe& p) {
  if (p.ready) return true;
  if (cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaStreamCreateWithFlags(&p.s_in2, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) != cudaSuccess) return false;
  cudaEvent_t* evs[9] = {&p.fork,        &p.loaded[0],   &p.loaded[1],   &p.loaded2[0], &p.loaded2[1],
                         &p.computed[0], &p.computed[1], &p.unloaded[0], &p.unloaded[1]};
  for (cudaEvent_t* e : evs)
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
  p.ready = true;
  return true;
}

size_t elem_size(wkv_dtype d) { return d == WKV_F32 ? 4 : 2; }

int64_t seg_len(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, int64_t seg_tokens) {
  if (seg_tokens > 0) return std::min<int64_t>(seg_tokens, std::max<int64_t>(T, 1));
  const int64_t per_token = std::max<int64_t>(1, B * C * 2 * (int64_t)elem_size(kv_dtype));
  int64_t s = std::max<int64_t>(64, kDefaultSegBytes / per_token / 64 * 64);
  return std::min<int64_t>(s, std::max<int64_t>(T, 1));
}

struct Layout {
  int64_t S;  // tokens per segment
  size_t k[2], v[2], o[2], carry, ws, ws_bytes, bytes;
};

bool layout(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, wkv_dtype out_dtype, int64_t seg_tokens,
            Layout* L) {
  if (B < 0 || T < 0 || C < 0 || seg_tokens < 0) return false;
  L->S = seg_len(B, T, C, kv_dtype, seg_tokens);
  const size_t kv = (size_t)(B * L->S * C) * elem_size(kv_dtype);
  const size_t ob = (size_t)(B * L->S * C) * elem_size(out_dtype);
  size_t off = 0;
  for (int i = 0; i < 2; ++i) {
    L->k[i] = off;
    off = round_up(off + kv, 256);
    L->v[i] = off;
    off = round_up(off + kv, 256);
    L->o[i] = off;
    off = round_up(off + ob, 256);
  }
  L->carry = off;
  off = round_up(off + 3 * sizeof(float) * (size_t)(B * C), 256);
  L->ws = off;
  // the forward's workspace for a full segment and for the (shorter) last one
  const int64_t last = T > 0 ? T - (T - 1) / L->S * L->S : 0;
  const size_t a = wkv_forward_workspace_size(B, L->S, C, nullptr);
  const size_t b = wkv_forward_workspace_size(B, last, C, nullptr);
  if (a == 0 && B * L->S * C > 0) return false;
  L->ws_bytes = std::max<size_t>(std::max(a, b), 256);
  L->bytes = L->ws + L->ws_bytes;
  return true;
}

}  // namespace

extern "C" {

size_t wkv_forward_host_buffer_size(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, wkv_dtype out_dtype,
                                    int64_t seg_tokens) {
  Layout L;
  if ((kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) || (out_dtype != WKV_F32 && out_dtype != WKV_BF16)) return 0;
  if (!layout(B, T, C, kv_dtype, out_dtype, seg_tokens, &L)) return 0;
  return L.bytes;
}

wkv_status wkv_forward_host(int64_t B, int64_t T, int64_t C, const void* k_host, const void* v_host,
                            wkv_dtype kv_dtype, const float* w, const float* u, void* out_host, wkv_dtype out_dtype,
                            const wkv_cstate* state_in, const wkv_state* state_out, void* dev_buffer,
                            size_t dev_bytes, int64_t seg_tokens, void* stream) {
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (out_dtype != WKV_F32 && out_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (kv_dtype == WKV_F32 && out_dtype != WKV_F32) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (seg_tokens < 0 || B < 0 || T < 0 || C < 0 || T >= (1ll << 24)) return WKV_ERR_INVALID_ARG;
  if (state_in && (!state_in->num || !state_in->den || !state_in->max_e)) return WKV_ERR_INVALID_ARG;
  if (state_out && (!state_out->num || !state_out->den || !state_out->max_e)) return WKV_ERR_INVALID_ARG;
  Layout L;
  if (!layout(B, T, C, kv_dtype, out_dtype, seg_tokens, &L)) return WKV_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B * T * C == 0) {
    // nothing to copy: wkv_forward handles the state (and checks the rest)
    return wkv_forward(B, T, C, k_host, v_host, kv_dtype, w, u, out_host, out_dtype, state_in, state_out,
                       dev_buffer, dev_bytes, stream, nullptr);
  }
  if (!k_host || !v_host || !out_host || !w || !u) return WKV_ERR_INVALID_ARG;
  if (!dev_buffer || reinterpret_cast<uintptr_t>(dev_buffer) % 256 != 0) return WKV_ERR_MISALIGNED;
  if (dev_bytes < L.bytes) return WKV_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
  HostPipe& P = g_pipe[dev];
  std::lock_guard<std::mutex> lk(P.mu);
  if (!pipe_ready(P)) return WKV_ERR_CUDA;

  unsigned char* db = static_cast<unsigned char*>(dev_buffer);
  const size_t kes = elem_size(kv_dtype), oes = elem_size(out_dtype);
  const int64_t nseg = (T + L.S - 1) / L.S;
  float* carry = reinterpret_cast<float*>(db + L.carry);
  const wkv_state carry_out = {carry, carry + B * C, carry + 2 * B * C};
  const wkv_cstate carry_in = {carry, carry + B * C, carry + 2 * B * C};
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  // the copies follow everything queued on the caller's stream before the call
  if (!ok(cudaEventRecord(P.fork, st)) || !ok(cudaStreamWaitEvent(P.s_in, P.fork, 0)) ||
      !ok(cudaStreamWaitEvent(P.s_in2, P.fork, 0)) || !ok(cudaStreamWaitEvent(P.s_out, P.fork, 0)))
    return WKV_ERR_CUDA;
  for (int64_t s = 0; s < nseg; ++s) {
    const int slot = (int)(s & 1);
    const int64_t t0 = s * L.S, len = std::min(L.S, T - t0);
    void* kd = db + L.k[slot];
    void* vd = db + L.v[slot];
    void* od = db + L.o[slot];
    // host -> device: rows of len*C elements at pitch T*C (one 2-D copy per
    // tensor, k and v on two streams: two copy engines share the link, which
    // is the limit either way: 21.6 against 21.7 ms per long-workload step);
    // the slot's buffers are free once the compute of segment s-2 ended
    if (s >= 2 && (!ok(cudaStreamWaitEvent(P.s_in, P.computed[slot], 0)) ||
                   !ok(cudaStreamWaitEvent(P.s_in2, P.computed[slot], 0))))
      return WKV_ERR_CUDA;
    const size_t wb = (size_t)(len * C) * kes, hp = (size_t)(T * C) * kes;
    if (!ok(cudaMemcpy2DAsync(kd, wb, static_cast<const unsigned char*>(k_host) + (size_t)(t0 * C) * kes, hp, wb,
                              (size_t)B, cudaMemcpyHostToDevice, P.s_in)) ||
        !ok(cudaMemcpy2DAsync(vd, wb, static_cast<const unsigned char*>(v_host) + (size_t)(t0 * C) * kes, hp, wb,
                              (size_t)B, cudaMemcpyHostToDevice, P.s_in2)) ||
        !ok(cudaEventRecord(P.loaded[slot], P.s_in)) || !ok(cudaEventRecord(P.loaded2[slot], P.s_in2)))
      return WKV_ERR_CUDA;
    // compute on the caller's stream, from the state after segment s-1
    if (!ok(cudaStreamWaitEvent(st, P.loaded[slot], 0)) || !ok(cudaStreamWaitEvent(st, P.loaded2[slot], 0)))
      return WKV_ERR_CUDA;
    if (s >= 2 && !ok(cudaStreamWaitEvent(st, P.unloaded[slot], 0))) return WKV_ERR_CUDA;
    const wkv_cstate* sin = s == 0 ? state_in : &carry_in;
    const wkv_state* sout = s == nseg - 1 ? state_out : &carry_out;
    const wkv_status r = wkv_forward(B, len, C, kd, vd, kv_dtype, w, u, od, out_dtype, sin, sout, db + L.ws,
                                     L.ws_bytes, stream, nullptr);
    if (r != WKV_OK) return r;
    if (!ok(cudaEventRecord(P.computed[slot], st))) return WKV_ERR_CUDA;
    // device -> host
    const size_t ob = (size_t)(len * C) * oes, op = (size_t)(T * C) * oes;
    if (!ok(cudaStreamWaitEvent(P.s_out, P.computed[slot], 0)) ||
        !ok(cudaMemcpy2DAsync(static_cast<unsigned char*>(out_host) + (size_t)(t0 * C) * oes, op, od, ob, ob,
                              (size_t)B, cudaMemcpyDeviceToHost, P.s_out)) ||
        !ok(cudaEventRecord(P.unloaded[slot], P.s_out)))
      return WKV_ERR_CUDA;
  }
  // the caller's stream ends after the last copy back (the copy streams are
  // in order, so the last event covers every earlier copy)
  if (!ok(cudaStreamWaitEvent(st, P.unloaded[(nseg - 1) & 1], 0))) return WKV_ERR_CUDA;
  return WKV_OK;
}

}  // extern "C"
