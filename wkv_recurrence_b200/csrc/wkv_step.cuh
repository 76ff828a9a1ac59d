// Batched one-token decode: S independent streams x C channels each take one
// token through the carried-state step of "Linear attention without writing a
// CUDA kernel", section "The recurrence".
//
// Purely elementwise and memory-bound (36 bytes per stream-channel in fp32:
// k, v, out, and the three state words read and written). Each thread owns VEC
// adjacent channels of one stream and moves them with 16-byte vector accesses.
//
// The state crosses HBM between steps as the page's triple (num, den, max_e),
// so the exponent is rounded once per step. To keep that rounding from adding
// up over many steps, the decayed exponent max_e - w is split into its fp32
// value md and the exact remainder r = (max_e - w) - md (Fast2Sum: md is the
// rounded difference and |w| is far below |max_e| whenever r matters); r is
// folded into the state as the factor e^r ~ 1 + r, or into the exponent of
// the incoming key when that key becomes the new maximum.
#pragma once

#include "wkv_device.cuh"

namespace wkv {

struct StepParams {
  long long n;  // S * C
  int C;
  const void* k;
  const void* v;
  const float* w;
  const float* u;
  void* out;
  const float* s_num;
  const float* s_den;
  const float* s_max;
  float* o_num;
  float* o_den;
  float* o_max;
  const float* w_t;  // this token's decay of every stream [S, C] in place of w, or NULL
  const void* r;     // receptance [S, C] (element type of k, v): out = sigmoid(r) wkv; or NULL
};

__device__ __forceinline__ void decode_token(float k, float v, float w, float u, float& num, float& den, float& m,
                                             float& out) {
  if (!(m > kNegBig)) m = kNegBig;  // empty state (-inf, or never written)
  // output: the state and the bonus-weighted token, relative to the larger
  // of the two exponents (one exponential; the other weight is exactly 1)
  const float D = (k + u) - m;
  const float x = ex2(-fabsf(D) * kLog2e);
  const bool tok = D > 0.f;
  const float a = tok ? x : 1.f;
  const float b = tok ? 1.f : x;
  out = fmaf(a, num, b * v) * rcp(fmaf(a, den, b));
  // advance: decay by w, add the token without the bonus
  const float md = m - w;
  const float r = (m - md) - w;          // (m - w) == md + r exactly
  const float D2 = (k - md) - r;         // k - (m - w)
  const float x2 = ex2(-fabsf(D2) * kLog2e);
  if (D2 > 0.f) {  // the key is the new maximum
    num = fmaf(x2, num, v);
    den = fmaf(x2, den, 1.f);
    m = k;
  } else {
    num = fmaf(x2, v, fmaf(num, r, num));
    den = fmaf(den, r, den) + x2;
    m = md;
  }
}

template <typename KV, typename OUT, int VEC>
__global__ void __launch_bounds__(256) wkv_step_kernel(const StepParams p) {
  const long long i0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * VEC;
  if (i0 >= p.n) return;
  const int c0 = (int)(i0 % p.C);
  if (VEC > 1 && i0 + VEC <= p.n) {
    // VEC divides C here, so the VEC channels sit in one row
    float kx[VEC], vx[VEC], num[VEC], den[VEC], mx[VEC], o[VEC], w[VEC], u[VEC];
    load_vec<KV, VEC>(reinterpret_cast<const KV*>(p.k) + i0, kx);
    load_vec<KV, VEC>(reinterpret_cast<const KV*>(p.v) + i0, vx);
    load_vec<float, VEC>(p.s_num + i0, num);
    load_vec<float, VEC>(p.s_den + i0, den);
    load_vec<float, VEC>(p.s_max + i0, mx);
    if (p.w_t) {
      load_vec<float, VEC>(p.w_t + i0, w);
    } else {
      load_vec<float, VEC>(p.w + c0, w);
    }
    load_vec<float, VEC>(p.u + c0, u);
#pragma unroll
    for (int e = 0; e < VEC; ++e) decode_token(kx[e], vx[e], w[e], u[e], num[e], den[e], mx[e], o[e]);
    if (p.r) {
      float rx[VEC];
      load_vec<KV, VEC>(reinterpret_cast<const KV*>(p.r) + i0, rx);
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[e] = gate(o[e], rx[e]);
    }
    store_vec<OUT, VEC>(reinterpret_cast<OUT*>(p.out) + i0, o);
    store_vec<float, VEC>(p.o_num + i0, num);
    store_vec<float, VEC>(p.o_den + i0, den);
    store_vec<float, VEC>(p.o_max + i0, mx);
  } else {
    for (int e = 0; e < VEC && i0 + e < p.n; ++e) {
      const long long i = i0 + e;
      const int c = (int)(i % p.C);
      float num = p.s_num[i], den = p.s_den[i], mx = p.s_max[i], o;
      const float kk = Elem<KV>::to_f32(reinterpret_cast<const KV*>(p.k)[i]);
      const float vv = Elem<KV>::to_f32(reinterpret_cast<const KV*>(p.v)[i]);
      decode_token(kk, vv, p.w_t ? p.w_t[i] : p.w[c], p.u[c], num, den, mx, o);
      if (p.r) o = gate(o, Elem<KV>::to_f32(reinterpret_cast<const KV*>(p.r)[i]));
      reinterpret_cast<OUT*>(p.out)[i] = Elem<OUT>::from_f32(o);
      p.o_num[i] = num;
      p.o_den[i] = den;
      p.o_max[i] = mx;
    }
  }
}

// Writes the empty state (0, 0, -inf) to n entries (a T = 0 forward with no
// state in).
__global__ void wkv_fill_empty_state(long long n, float* num, float* den, float* mx) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    num[i] = 0.f;
    den[i] = 0.f;
    mx[i] = -__int_as_float(0x7f800000);
  }
}

}  // namespace wkv
