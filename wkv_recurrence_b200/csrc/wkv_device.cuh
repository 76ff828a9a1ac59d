// Device-side building blocks of the WKV kernels: PTX wrappers (mbarrier, TMA,
// global timer, fast exp2 / reciprocal), vector loads and stores for fp32 and
// bf16 rows, and the per-token arithmetic of the recurrence in the anchored
// form described below.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv {

constexpr float kLog2e = 1.4426950408889634f;
// Exponent that stands for "no state yet" (-inf on the API). Finite so that
// differences of two empty exponents stay finite; e^{x - kNegBig} underflows.
constexpr float kNegBig = -1.0e30f;
// Upper clamp of the output's bonus exponent, natural units. e^44 ~ 2^63.5, so
// the clamped weight times any |v| < 2^64 stays finite while den (>= 1 and at
// most a few million for any state this library produces) is negligible next
// to it when the clamp is active.
constexpr float kBonusClamp = 44.0f;

// device-side status bits, kept in the workspace header
constexpr uint32_t kStatusWaitTimeout = 1u;
constexpr uint32_t kStatusBoundsError = 2u;  // bounds-checked build only

struct WsHeader {
  uint32_t ticket;   // next tile to hand out (chunked kernel)
  uint32_t done;     // CTAs that finished (chunked kernel)
  uint32_t epoch;    // number of completed chunked launches on this workspace
  uint32_t status;   // OR of kStatus* bits since the last wkv_query_status
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

// ---------------------------------------------------------------------------
// Index checks of the bounds-checked build (compiled with -DWKV_DEBUG): an
// index outside its array sets kStatusBoundsError in the status word of the
// call's workspace header and the access is skipped; nothing traps, so the
// context stays usable and wkv_query_status reports it. In the ordinary build
// every check is the constant true and compiles away.
// ---------------------------------------------------------------------------
#ifdef WKV_DEBUG
__device__ __forceinline__ bool dbg_ok(WsHeader* h, bool in_bounds) {
  if (!in_bounds && h) atomicOr(&h->status, kStatusBoundsError);
  return in_bounds;
}
#define WKV_IN(h, i, n) ::wkv::dbg_ok((h), (unsigned long long)(i) < (unsigned long long)(n))
#else
#define WKV_IN(h, i, n) true
#endif

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tests whether the phase with the given parity has completed. If it has not,
// the thread may be suspended (without taking issue slots) until it completes
// or for at most kSuspendHintNs.
constexpr uint32_t kSuspendHintNs = 100000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most
// timeout_ns. Returns false if the limit was reached.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// 3-D tiled TMA load of the box at (c0, c1, c2) into shared memory, completing
// on `bar`. c0 (the contiguous coordinate) times the element size must be a
// multiple of 16 bytes; callers pass channel offsets that are multiples of the
// channel-group width (>= 32 channels).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ld_relaxed_f4(const float4* p) {
  float4 r;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p)
               : "memory");
  return r;
}

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  __device__ __forceinline__ static float to_f32(float x) { return x; }
  __device__ __forceinline__ static float from_f32(float x) { return x; }
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// VEC consecutive elements -> fp32 registers. `p` is aligned to VEC elements.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&x)[VEC]);

template <>
__device__ __forceinline__ void load_vec<float, 1>(const float* p, float (&x)[1]) { x[0] = *p; }
template <>
__device__ __forceinline__ void load_vec<float, 2>(const float* p, float (&x)[2]) {
  float2 a = *reinterpret_cast<const float2*>(p);
  x[0] = a.x; x[1] = a.y;
}
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&x)[4]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
__device__ __forceinline__ void unpack_bf16x2(uint32_t u, float& lo, float& hi) {
  lo = __uint_as_float(u << 16);
  hi = __uint_as_float(u & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 1>(const __nv_bfloat16* p, float (&x)[1]) {
  x[0] = __bfloat162float(*p);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 2>(const __nv_bfloat16* p, float (&x)[2]) {
  unpack_bf16x2(*reinterpret_cast<const uint32_t*>(p), x[0], x[1]);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&x)[4]) {
  uint2 a = *reinterpret_cast<const uint2*>(p);
  unpack_bf16x2(a.x, x[0], x[1]);
  unpack_bf16x2(a.y, x[2], x[3]);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&x)[8]) {
  uint4 a = *reinterpret_cast<const uint4*>(p);
  unpack_bf16x2(a.x, x[0], x[1]);
  unpack_bf16x2(a.y, x[2], x[3]);
  unpack_bf16x2(a.z, x[4], x[5]);
  unpack_bf16x2(a.w, x[6], x[7]);
}

template <typename T, int VEC>
__device__ __forceinline__ void store_vec(T* p, const float (&x)[VEC]);

template <>
__device__ __forceinline__ void store_vec<float, 1>(float* p, const float (&x)[1]) { *p = x[0]; }
template <>
__device__ __forceinline__ void store_vec<float, 2>(float* p, const float (&x)[2]) {
  *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 1>(__nv_bfloat16* p, const float (&x)[1]) {
  *p = __float2bfloat16_rn(x[0]);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 2>(__nv_bfloat16* p, const float (&x)[2]) {
  *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&x)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 8>(__nv_bfloat16* p, const float (&x)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                            pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}

// Streaming stores (evict-first in L2). `p` is aligned to VEC elements.
template <typename T, int VEC>
__device__ __forceinline__ void stg_stream(T* p, const float (&x)[VEC]);

template <>
__device__ __forceinline__ void stg_stream<float, 1>(float* p, const float (&x)[1]) {
  asm volatile("st.global.cs.f32 [%0], %1;" ::"l"(p), "f"(x[0]) : "memory");
}
template <>
__device__ __forceinline__ void stg_stream<float, 2>(float* p, const float (&x)[2]) {
  asm volatile("st.global.cs.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(x[0]), "f"(x[1]) : "memory");
}
template <>
__device__ __forceinline__ void stg_stream<float, 4>(float* p, const float (&x)[4]) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(x[0]), "f"(x[1]), "f"(x[2]),
               "f"(x[3])
               : "memory");
}
template <>
__device__ __forceinline__ void stg_stream<__nv_bfloat16, 1>(__nv_bfloat16* p, const float (&x)[1]) {
  *p = __float2bfloat16_rn(x[0]);
}
template <>
__device__ __forceinline__ void stg_stream<__nv_bfloat16, 2>(__nv_bfloat16* p, const float (&x)[2]) {
  asm volatile("st.global.cs.b32 [%0], %1;" ::"l"(p), "r"(pack_bf16x2(x[0], x[1])) : "memory");
}
template <>
__device__ __forceinline__ void stg_stream<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&x)[4]) {
  asm volatile("st.global.cs.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(pack_bf16x2(x[0], x[1])),
               "r"(pack_bf16x2(x[2], x[3]))
               : "memory");
}

// ---------------------------------------------------------------------------
// The recurrence in anchored form
// ---------------------------------------------------------------------------
//
// The page's state is (num, den, max_e) with the true pair N = num e^{max_e},
// D = den e^{max_e}. Each token decays max_e by w. Done literally in fp32,
// max_e - w is rounded every token, and when |max_e| >> w that rounding error
// has the same sign token after token, so the effective decay drifts (several
// percent of the decay rate for max_e ~ 60, w ~ 1e-4).
//
// These kernels keep the exponent as an ANCHOR plus a COUNT: `ma` is the
// exponent of the token that last became the maximum (a key k_i, exact), and
// `nf` is the number of decays since then, so max_e = ma - nf*w is formed by
// one fma from exact operands and its rounding never accumulates. While no new
// key exceeds the decayed maximum, num and den are left alone (the page's
// factor exp(max_e - w - e') is exactly 1 then) and only the count moves.
//
// Invariant: den >= 1 for a non-empty state (the anchor token contributes
// exactly 1), which lets the output use one clamped exponential instead of a
// compare-and-select of two (see out_token).
struct Acc {
  float num, den, ma, nf;
};

__device__ __forceinline__ Acc acc_empty() { return Acc{0.f, 0.f, kNegBig, 0.f}; }

__device__ __forceinline__ float acc_max_e(const Acc& s, float w) { return fmaf(-s.nf, w, s.ma); }

// wkv for one token from the state before it: the state pair plus the current
// token with weight e^{u+k}, both relative to the state's max exponent M.
// beta = e^{k+u-M} is clamped at e^44: when the clamp is active the current
// token outweighs the state by more than 2^63 and the result is v to within
// den * 2^-63.
__device__ __forceinline__ float out_token(const Acc& s, float k, float v, float w, float u) {
  const float M = fmaf(-s.nf, w, s.ma);
  const float D = (k + u) - M;
  const float beta = ex2(fminf(D, kBonusClamp) * kLog2e);
  return fmaf(beta, v, s.num) * rcp(s.den + beta);
}

// Decays the state by one token and adds token (k, v) with weight e^{k}.
__device__ __forceinline__ void add_token(Acc& s, float k, float v, float w) {
  const float nf1 = s.nf + 1.f;
  const float Md = fmaf(-nf1, w, s.ma);  // max exponent after the decay
  const float D2 = k - Md;
  const float x = ex2(-fabsf(D2) * kLog2e);
  const bool reset = k > Md;  // the new key becomes the maximum (and the anchor)
  const float a = reset ? x : 1.f;
  const float b = reset ? 1.f : x;
  s.num = fmaf(a, s.num, b * v);
  s.den = fmaf(a, s.den, b);
  s.ma = reset ? k : s.ma;
  s.nf = reset ? 0.f : nf1;
}

// Output and state advance for one token, with one exponential.
//
// Let Md be the state's max exponent after this token's decay and D2 = k - Md.
// The update needs e^{-|D2|} (the smaller of the two weights; the other is 1).
// The output compares the undecayed state (exponent Md + w) with the current
// token with its bonus (exponent k + u); dividing both weights by e^{w} makes
// them the update's weights, with the current token's multiplied by the
// per-channel constant c = e^{u-w}. So one ex2 serves both halves.
// Valid while c and 1/c stay far inside the fp32 range; callers take this
// path only when |u - w| <= kFastUW (else out_token + add_token).
constexpr float kFastUW = 40.0f;

__device__ __forceinline__ float step_token(Acc& s, float k, float v, float w, float c) {
  const float nf1 = s.nf + 1.f;
  const float Md = fmaf(-nf1, w, s.ma);
  const float D2 = k - Md;
  const float x = ex2(-fabsf(D2) * kLog2e);
  const bool reset = k > Md;            // the key is the new maximum (and anchor)
  const float a = reset ? x : 1.f;      // weight of the carried state
  const float b = reset ? 1.f : x;      // weight of the current token (no bonus)
  const float bc = b * c;               // ... and with the bonus
  const float out = fmaf(bc, v, a * s.num) * rcp(fmaf(a, s.den, bc));
  s.num = fmaf(a, s.num, b * v);
  s.den = fmaf(a, s.den, b);
  s.ma = reset ? k : s.ma;
  s.nf = reset ? 0.f : nf1;
  return out;
}

__device__ __forceinline__ bool fast_uw(float u, float w) { return fabsf(u - w) <= kFastUW; }

// step_token over N consecutive tokens of VEC channels, reorganised for
// instruction-level parallelism. Only the anchor and count are carried from
// token to token through a short chain (fma, compare, select), and only it
// runs first, for all N tokens; the exponentials, the num/den updates
// and the outputs of the N tokens then have no dependency on each other
// beyond one fma per token, so their latencies overlap. Every token goes
// through exactly the operations of step_token, in the same order, so the
// results are bitwise the same.
template <int N, int VEC>
__device__ __forceinline__ void step_tokens(Acc (&s)[VEC], const float (&k)[N][VEC], const float (&v)[N][VEC],
                                            const float (&w)[VEC], const float (&c)[VEC], float (&out)[N][VEC]) {
  float d2[N][VEC];
  bool rs[N][VEC];
  // The chain carries the anchor and cnt = (decays since the anchor) + 1, so
  // that per token it is one fma, one compare and one select; the count's
  // increment and the difference k - Md stay off it.
  float cnt[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) cnt[e] = s[e].nf + 1.f;
#pragma unroll
  for (int i = 0; i < N; ++i) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float Md = fmaf(-cnt[e], w[e], s[e].ma);
      rs[i][e] = k[i][e] > Md;
      d2[i][e] = k[i][e] - Md;
      s[e].ma = rs[i][e] ? k[i][e] : s[e].ma;
      cnt[e] = rs[i][e] ? 1.f : cnt[e] + 1.f;
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) s[e].nf = cnt[e] - 1.f;
#pragma unroll
  for (int i = 0; i < N; ++i) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float x = ex2(-fabsf(d2[i][e]) * kLog2e);
      const float a = rs[i][e] ? x : 1.f;
      const float b = rs[i][e] ? 1.f : x;
      const float bc = b * c[e];
      out[i][e] = fmaf(bc, v[i][e], a * s[e].num) * rcp(fmaf(a, s[e].den, bc));
      s[e].num = fmaf(a, s[e].num, b * v[i][e]);
      s[e].den = fmaf(a, s[e].den, b);
    }
  }
}

// Associative combine: `a` covers the tokens before `b`, and `b` spans len_b
// tokens. The result covers both: `a` is decayed across b's tokens (its count
// grows by len_b) and the two are added relative to the larger exponent, which
// becomes the anchor. The empty state is the identity.
// The exponent difference (a.ma - na w) - (b.ma - b.nf w) is formed as
// (a.ma - b.ma) - (na - b.nf) w: the counts are integers (exact), the anchors
// are keys of similar size (their difference is often exact), so it is rounded
// about once, at its own magnitude, instead of twice at the magnitude of the
// anchored exponents (long chains of combines, as in a scan of many chunk
// totals, keep their accuracy).
__device__ __forceinline__ Acc combine(const Acc& a, const Acc& b, float len_b, float w) {
  const float na = a.nf + len_b;
  const float d = fmaf(-(na - b.nf), w, a.ma - b.ma);
  const bool a_wins = d >= 0.f;
  const float s = ex2(-fabsf(d) * kLog2e);
  Acc r;
  r.num = a_wins ? fmaf(s, b.num, a.num) : fmaf(s, a.num, b.num);
  r.den = a_wins ? fmaf(s, b.den, a.den) : fmaf(s, a.den, b.den);
  r.ma = a_wins ? a.ma : b.ma;
  r.nf = a_wins ? na : b.nf;
  return r;
}

// A caller's state triple -> anchored form. Empty when den <= 0, max_e is not
// above kNegBig (-inf included) or any value is NaN. A den outside [1, 2^24] is
// rescaled to 1 (moving log(den) into the exponent) so that the invariant
// den >= 1 holds and den stays small next to the output clamp.
__device__ __forceinline__ Acc acc_from_state(float num, float den, float max_e) {
  if (!(den > 0.f) || !(max_e > kNegBig) || num != num) return acc_empty();
  if (den < 1.f || den > 16777216.f) {
    const float inv = 1.f / den;
    const float lnden = lg2(den) * 0.6931471805599453f;
    return Acc{num * inv, 1.f, max_e + lnden, 0.f};
  }
  return Acc{num, den, max_e, 0.f};
}

// ---------------------------------------------------------------------------
// Per-token decay w_t ("RWKV-v6 Architecture", section "2. Dynamic
// Data-Dependent Decay"): the decay since the anchor is no longer count * w but
// a running sum of the tokens' decays. Acc.nf then holds that sum, and sums
// over many tokens are compensated (the rounding error of each addition is
// carried separately, Knuth's TwoSum), so that a long memory of small decays
// does not drift the way a plain fp32 running sum would.
// ---------------------------------------------------------------------------

// hi + lo = a + b exactly, hi = fl(a + b) (Knuth's TwoSum, no precondition on
// the magnitudes)
__device__ __forceinline__ void two_sum(float a, float b, float& hi, float& lo) {
  hi = a + b;
  const float bp = hi - a;
  lo = (a - (hi - bp)) + (b - bp);
}

// Combine with per-token decays: `b` covers tokens whose decays sum to w_b, so
// `a` is decayed by w_b across them. Same structure as combine().
__device__ __forceinline__ Acc combine_wt(const Acc& a, const Acc& b, float w_b) {
  const float na = a.nf + w_b;
  const float d = (a.ma - b.ma) - (na - b.nf);
  const bool a_wins = d >= 0.f;
  const float s = ex2(-fabsf(d) * kLog2e);
  Acc r;
  r.num = a_wins ? fmaf(s, b.num, a.num) : fmaf(s, a.num, b.num);
  r.den = a_wins ? fmaf(s, b.den, a.den) : fmaf(s, a.den, b.den);
  r.ma = a_wins ? a.ma : b.ma;
  r.nf = a_wins ? na : b.nf;
  return r;
}

// One token with its own decay wt: output from the state before it (with the
// bonus u), then the advance (decay by e^{-wt}, add the token without bonus).
// `lo` carries the compensation of the running decay sum s.nf; it is reset
// with the anchor.
__device__ __forceinline__ float step_token_wt(Acc& s, float& lo, float k, float v, float wt, float u) {
  // output: the undecayed state (exponent ma - nf - lo) against k + u
  const float M = (s.ma - s.nf) - lo;
  const float D = (k + u) - M;
  const float beta = ex2(fminf(D, kBonusClamp) * kLog2e);
  const float out = fmaf(beta, v, s.num) * rcp(s.den + beta);
  // advance
  float hi, e;
  two_sum(s.nf, wt, hi, e);
  const float lo1 = lo + e;
  const float Md = (s.ma - hi) - lo1;
  const float D2 = k - Md;
  const float x = ex2(-fabsf(D2) * kLog2e);
  const bool reset = D2 > 0.f;
  const float a = reset ? x : 1.f;
  const float b = reset ? 1.f : x;
  s.num = fmaf(a, s.num, b * v);
  s.den = fmaf(a, s.den, b);
  s.ma = reset ? k : s.ma;
  s.nf = reset ? 0.f : hi;
  lo = reset ? 0.f : lo1;
  return out;
}

// The state's max exponent with per-token decays (ma - nf, and the
// compensation of nf).
__device__ __forceinline__ float acc_max_e_wt(const Acc& s, float lo) { return (s.ma - s.nf) - lo; }

// ---------------------------------------------------------------------------
// The receptance gate of the Time-Mixing block: y = sigmoid(r) * wkv.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float gate(float y, float r) { return y * rcp(1.f + ex2(-r * kLog2e)); }

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, barrier, and loads from another CTA's shared
// memory (distributed shared memory).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// (the non-.aligned forms: callers need not be converged)
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }
// shared-memory address of the same variable in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t map_shared_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float4 acc_pack(const Acc& s) { return make_float4(s.num, s.den, s.ma, s.nf); }
__device__ __forceinline__ Acc acc_unpack(const float4& f) { return Acc{f.x, f.y, f.z, f.w}; }

}  // namespace wkv
