// Backward of the WKV forward: the gradients of a loss L with respect to k, v,
// w, u and the state passed in, given g = dL/d wkv for every output (no loss
// term on the final state).
//
// The chain rule through the step function of "Linear attention without
// writing a CUDA kernel", section "The recurrence", run backwards in time.
// With the state before token t as the pair (N_t, D_t) and the output
// wkv_t = A_t / Z_t, A_t = N_t + e^{u+k_t} v_t, Z_t = D_t + e^{u+k_t}, the
// reverse accumulators dN_t = dL/dN_t and dD_t = dL/dD_t obey
//     dN_t = g_t / Z_t + e^{-w} dN_{t+1},   dD_t = -g_t wkv_t / Z_t + e^{-w} dD_{t+1},
// a linear recurrence of exactly the forward's shape running the other way:
// its "keys" are -M_t (M_t the largest exponent in Z_t) and its two value
// streams are p_t = g_t / z_t and q_t = -g_t wkv_t / z_t (z_t = Z_t e^{-M_t}).
// So the reverse accumulators use the same anchored arithmetic (Acc: num and
// den hold the two value streams, the anchor and count give their exponent)
// and the same associative combine. Then, with R = (dN_{t+1}, dD_{t+1}):
//     dv_t = g_t e^{u+k_t} / Z_t + e^{k_t} dN_{t+1}
//     dk_t = g_t e^{u+k_t} (v_t - wkv_t) / Z_t + e^{k_t} (v_t dN_{t+1} + dD_{t+1})
//     du  += g_t e^{u+k_t} (v_t - wkv_t) / Z_t
//     dw  -= e^{-w} (N_t dN_{t+1} + D_t dD_{t+1})
// and dnum0 = e^{m0} dN_0, dden0 = e^{m0} dD_0, dm0 = num0 dnum0 + den0 dden0.
//
// The work is cut into chunks of L tokens like the forward's three-launch
// scan, so that every pass is parallel over (batch row, chunk, channel):
//   A, S  the forward's chunk totals and their scan: the forward state
//         entering every chunk (x0);
//   R1    wkv_bwd_rev_totals: per chunk, the forward replayed from x0 and the
//         chunk's reverse aggregate (its tokens' contributions to dN, dD at
//         the chunk's start);
//   RS    the scan of R1's aggregates from the last chunk backwards: the
//         reverse state entering every chunk from its end (rin);
//   R2    wkv_bwd_chunk: per chunk, the forward replayed from x0 (states kept
//         at every 4th token in registers, the others recomputed), then the
//         tokens in reverse from rin, writing dk, dv and per-chunk partial sums
//         of du, dw; chunk 0 also yields the state gradients;
//   RED   wkv_bwd_reduce: du, dw as compensated sums of the partials over the
//         chunks and batch rows (a warp per channel), in a fixed order.
// One 32-thread CTA per (batch row, chunk, 32 channels) in R1 and R2, the
// chunk's k, v and g copied into shared memory by TMA. All orders of
// accumulation depend on the shape only, so results are bitwise reproducible.
#pragma once

#include "wkv_device.cuh"
#include "wkv_fwd.cuh"

namespace wkv {

struct BwdParams {
  int B, T, C;
  int NG;            // 64-channel groups per batch row (layout of x0, rtot, rin)
  int nch;           // chunks per sequence
  int chunk_len;
  const void* k;
  const void* v;
  const float* w;
  const float* u;
  const float* g;    // dL/d wkv [B, T, C] fp32
  const float* s_num;  // state in (NULL = empty)
  const float* s_den;
  const float* s_max;
  float* dk;         // [B, T, C] fp32
  float* dv;
  float* dw;         // [C] fp32
  float* du;
  float* d_num;      // [B, C] state gradients (NULL = not written)
  float* d_den;
  float* d_max;
  const float4* x0;  // forward state entering every chunk [nch][B*NG][64]
  float4* rtot;      // reverse aggregate of every chunk [nch][B*NG][64] (chunk 0 unused)
  float4* rin;       // reverse state entering every chunk from its end [nch][B*NG][64]
  float* pdw;        // per-chunk partial sums [nch][B][C]
  float* pdu;
  WsHeader* hdr;     // status word: wait timeouts (and index errors in the bounds-checked build)
  uint64_t timeout_ns;
};

__device__ __forceinline__ size_t bwd_slot(const BwdParams& p, int j, int b, int c) {
  return ((size_t)j * p.B * p.NG + (size_t)b * p.NG + c / 64) * 64 + c % 64;
}

// Exponents are kept ANCHORED, as in the forward: never as one rounded fp32
// number of large magnitude, but as an exact key plus integer multiples of w
// (and, for the output's largest exponent, possibly u), so that the difference
// of two exponents -- the only thing an exponential here ever needs -- is
// formed at its own magnitude. (With keys of +-60 and the reverse exponents
// near -60, rounding the exponents themselves would cost ~1e-5 of relative
// accuracy per gradient.)
//
// The output's largest exponent of token t is M_t = max(m_t, k_t + u) with
// m_t = ma - nf w the state's: anchored as (key, uf, cnt) with
// M_t = key - cnt w + uf u, either (ma, 0, nf) or (k_t, 1, 0).
struct OutStat {
  float key, uf, cnt;  // M_t = key - cnt w + uf u
  float z;             // Z_t e^{-M_t} (>= 1)
  float b;             // e^{u + k_t - M_t}, the current token's weight
  float out;           // wkv_t
};

// e^{x} for an exponent given as the unevaluated sum x = hi + lo: 2^{hi log2 e}
// with the product's rounding error recovered by an fma and the low parts
// applied as the first-order factor 1 + (...) ln 2 (|lo| is below 2^-20 of
// |hi|, so the second-order term is far below fp32 resolution).
constexpr float kLog2eLo = 1.925963e-8f;  // log2(e) minus its nearest fp32 value
constexpr float kLn2 = 0.69314718f;
__device__ __forceinline__ float exp_hl(float hi, float lo) {
  const float y = hi * kLog2e;
  const float yl = fmaf(hi, kLog2e, -y) + fmaf(hi, kLog2eLo, lo * kLog2e);
  const float r = ex2(y);
  return fmaf(r, yl * kLn2, r);
}

// The exponent n w + (a - b) + c as hi + lo with no rounding lost: TwoSum
// (Knuth) for the additions and the fma-based TwoProduct (Ogita, Rump and
// Oishi, "Accurate sum and dot product", 2005) for n w. Gradients that are a
// single exponential of an exponent near +-60 need this: rounding the
// exponent to fp32 would cost |x| 2^-24 ~ 4e-6 of relative accuracy per
// operation, several of which would exceed the 1e-5 bar.
__device__ __forceinline__ void exponent_hl(float n, float w, float a, float b, float c, float& hi, float& lo) {
  float s1, e1, s2, e2, e3;
  two_sum(a, -b, s1, e1);
  two_sum(s1, c, s2, e2);
  const float pr = n * w;
  const float ep = fmaf(n, w, -pr);
  two_sum(s2, pr, hi, e3);
  lo = (e1 + e2) + (ep + e3);
}
__device__ __forceinline__ float exp_exact(float n, float w, float a, float b, float c) {
  float hi, lo;
  exponent_hl(n, w, a, b, c, hi, lo);
  return exp_hl(hi, lo);
}

// kExact: the current token's weight b = e^{D} (D < 0) evaluated from the
// exact exponent (the gradient pass, where b multiplies dk and dv directly);
// otherwise rounded like everywhere else.
// Exponents of magnitude up to kExactFrom are evaluated rounded: a few
// roundings at that magnitude cost at most ~2e-6 of relative accuracy. A warp
// takes the exact evaluation when any of its lanes has a larger one.
constexpr float kExactFrom = 8.0f;

// (mask: the lanes of the warp taking part, for the kExact vote.)
template <bool kExact = false>
__device__ __forceinline__ OutStat out_stat(const Acc& s, float k, float v, float u, float w,
                                            unsigned mask = 0xffffffffu) {
  // D = (k + u) - m, formed as (k - ma) + u + nf w
  float D = fmaf(s.nf, w, (k - s.ma) + u);
  float x;
  if (kExact && __any_sync(mask, fabsf(D) > kExactFrom)) {
    float Dlo;
    exponent_hl(s.nf, w, k, s.ma, u, D, Dlo);
    x = exp_hl(-fabsf(D), D > 0.f ? -Dlo : Dlo);
  } else {
    x = ex2(-fabsf(D) * kLog2e);
  }
  const bool tok = D > 0.f;  // the current token carries the largest exponent
  const float a = tok ? x : 1.f;
  const float b = tok ? 1.f : x;
  OutStat o;
  o.key = tok ? k : s.ma;
  o.uf = tok ? 1.f : 0.f;
  o.cnt = tok ? 0.f : s.nf;
  o.z = fmaf(a, s.den, b);
  o.out = fmaf(a, s.num, b * v) * rcp(o.z);
  o.b = b;
  return o;
}

// A reverse accumulator (dN, dD) = (rn, rd) e^{Q} at some position, with
// Q = -qk - qu u + qc w: the anchor token's -M (qk its key, qu its u flag) and
// qc = its count minus its distance from the position (an integer).
struct RAcc {
  float rn, rd, qk, qc, qu;
};

constexpr float kPosBig = 1.0e30f;  // qk of the empty accumulator (Q = -1e30)

__device__ __forceinline__ RAcc racc_empty() { return RAcc{0.f, 0.f, kPosBig, 0.f, 0.f}; }

// Packed as a float4: qc + qu / 2 in the last slot (qc is an integer below
// 2^22 in magnitude, so the half is exact).
__device__ __forceinline__ float4 racc_pack(const RAcc& r) { return make_float4(r.rn, r.rd, r.qk, r.qc + 0.5f * r.qu); }
__device__ __forceinline__ RAcc racc_unpack(const float4& f) {
  const float qc = floorf(f.w);
  return RAcc{f.x, f.y, f.z, qc, 2.f * (f.w - qc)};
}

// Adds a token whose exponent at the accumulator's position is
// -key - uf u + cnt w, with value streams (p, q).
__device__ __forceinline__ void racc_add(RAcc& r, float key, float uf, float cnt, float p, float q, float w,
                                         float u) {
  const float d = fmaf(cnt - r.qc, w, (r.qk - key) + (r.qu - uf) * u);  // token's exponent - Q
  const float x = ex2(-fabsf(d) * kLog2e);
  const bool tok = d > 0.f;
  const float a = tok ? x : 1.f;
  const float bb = tok ? 1.f : x;
  r.rn = fmaf(a, r.rn, bb * p);
  r.rd = fmaf(a, r.rd, bb * q);
  r.qk = tok ? key : r.qk;
  r.qu = tok ? uf : r.qu;
  r.qc = tok ? cnt : r.qc;
}

// `a` stands `len` tokens after `b`'s position (it covers the tokens after
// b's): moved to b's position and merged. Associative, the empty accumulator
// is the identity.
__device__ __forceinline__ RAcc racc_combine(const RAcc& a, const RAcc& b, float len, float w, float u) {
  const float ac = a.qc - len;
  const float d = fmaf(ac - b.qc, w, (b.qk - a.qk) + (b.qu - a.qu) * u);  // a's exponent - b's
  const bool a_wins = d >= 0.f;
  const float s = ex2(-fabsf(d) * kLog2e);
  RAcc r;
  r.rn = a_wins ? fmaf(s, b.rn, a.rn) : fmaf(s, a.rn, b.rn);
  r.rd = a_wins ? fmaf(s, b.rd, a.rd) : fmaf(s, a.rd, b.rd);
  r.qk = a_wins ? a.qk : b.qk;
  r.qu = a_wins ? a.qu : b.qu;
  r.qc = a_wins ? ac : b.qc;
  return r;
}


// The chunk's tiles in shared memory: k, v (element type KV) and g (fp32), L
// tokens x 32 channels each, copied by TMA on one mbarrier. Returns false if
// the copy did not land within the wait limit (the status word is set).
// (Measured: reading g from global memory a few tokens ahead instead, for
// more resident CTAs, was slower overall.)
template <typename KV, int L>
__host__ __device__ constexpr uint32_t bwd_tile_bytes() {
  return (uint32_t)(L * 32 * (2 * sizeof(KV) + sizeof(float)));
}

template <typename KV, int L>
__device__ __forceinline__ bool bwd_load_tile(const BwdParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                                              const CUtensorMap* tg, unsigned char* smem, uint64_t* bar, int gw,
                                              int t0, int b) {
  KV* ks = reinterpret_cast<KV*>(smem);
  if ((threadIdx.x & 31) == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, bwd_tile_bytes<KV, L>());
    tma_load_3d(ks, tk, bar, gw * 32, t0, b);
    tma_load_3d(ks + L * 32, tv, bar, gw * 32, t0, b);
    tma_load_3d(reinterpret_cast<float*>(ks + 2 * L * 32), tg, bar, gw * 32, t0, b);
  }
  __syncwarp();
  const bool ok = mbar_wait(bar, 0, p.timeout_ns);
  if (!ok && (threadIdx.x & 31) == 0) {
    atomicOr(&p.hdr->status, kStatusWaitTimeout);
    (void)mbar_wait(bar, 0, p.timeout_ns);  // bounded drain
  }
  return __all_sync(0xffffffffu, ok);
}

// R1. One 32-thread CTA per (batch row, chunk j >= 1, 32 channels). The
// forward is replayed from x0[j] out of the chunk's tiles to get M_t, z_t,
// wkv_t of every token; the chunk's reverse aggregate (relative to its first
// token: token t enters with exponent -M_t - (t - t0) w) is folded in token
// order.
template <typename KV, int L>
__global__ void __launch_bounds__(32)
    wkv_bwd_rev_totals(const BwdParams p, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmg) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const KV* ks = reinterpret_cast<const KV*>(smem);
  const KV* vs = ks + L * 32;
  const float* gs = reinterpret_cast<const float*>(vs + L * 32);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + bwd_tile_bytes<KV, L>());
  const int lane = threadIdx.x;
  const int ngw = (p.C + 31) / 32;
  const long long item = blockIdx.x;
  const int gw = (int)(item % ngw);
  const int j = 1 + (int)((item / ngw) % (p.nch - 1));
  const int b = (int)(item / ((long long)ngw * (p.nch - 1)));
  const int t0 = j * L;
  if (!bwd_load_tile<KV, L>(p, &tmk, &tmv, &tmg, smem, bar, gw, t0, b)) return;
  const int c = gw * 32 + lane;
  if (c >= p.C) return;
  const float w = __ldg(p.w + c), u = __ldg(p.u + c);
  Acc s = acc_unpack(p.x0[bwd_slot(p, j, b, c)]);
  const int n = min(L, p.T - t0);
  RAcc r = racc_empty();  // at the chunk's first token
  for (int t = 0; t < n; ++t) {
    const float k = Elem<KV>::to_f32(ks[t * 32 + lane]), v = Elem<KV>::to_f32(vs[t * 32 + lane]);
    const float g = gs[t * 32 + lane];
    const OutStat o = out_stat(s, k, v, u, w);
    const float rz = rcp(o.z);
    // token t's exponent at the chunk's start: -M_t - t w
    racc_add(r, o.key, o.uf, o.cnt - (float)t, g * rz, -g * o.out * rz, w, u);
    add_token(s, k, v, w);
  }
  if (WKV_IN(p.hdr, bwd_slot(p, j, b, c), (size_t)p.nch * p.B * p.NG * 64)) p.rtot[bwd_slot(p, j, b, c)] = racc_pack(r);
}

// RS. The reverse scan of the chunks' reverse aggregates: rin[j] = the reverse
// state at the end of chunk j from every later chunk (rin[nch-1] empty),
// rin[j] = combine(rin[j+1], rtot[j+1]) with rin[j+1] decayed across chunk
// j+1. Same two-level structure as the forward's wkv_tile_scan (16 channels x
// SEG segments per CTA, segments of about 16 chunks), walking the chunks from
// the last: index q stands for chunk nch-1-q.
template <int SEG>
__global__ void __launch_bounds__(16 * SEG) wkv_bwd_rev_scan(const BwdParams p) {
  constexpr int CH = 16;
  __shared__ float4 seg_st[SEG][CH];
  const int bg = blockIdx.x >> 2;
  const int ch = threadIdx.x % CH;
  const int cl = (blockIdx.x & 3) * CH + ch;
  const int sg = threadIdx.x / CH;
  const int b = bg / p.NG, c = (bg % p.NG) * 64 + cl;
  const float w = c < p.C ? __ldg(p.w + c) : 0.f;
  const float u = c < p.C ? __ldg(p.u + c) : 0.f;
  const int ntot = p.nch - 1;  // aggregates of chunks nch-1 .. 1
  const int per = (ntot + SEG - 1) / SEG;
  const int q0 = min(ntot, sg * per), q1 = min(ntot, q0 + per);
  const float fL = (float)p.chunk_len;
  auto tot = [&](int q) { return racc_unpack(p.rtot[bwd_slot(p, p.nch - 1 - q, b, c)]); };
  // 1. this segment's aggregate
  RAcc t = racc_empty();
  if (c < p.C)
    for (int q = q0; q < q1; ++q) t = racc_combine(t, tot(q), fL, w, u);
  seg_st[sg][ch] = racc_pack(t);
  __syncthreads();
  // 2. the state entering every segment
  if (sg == 0) {
    RAcc x = racc_empty();
    for (int k = 0; k < SEG; ++k) {
      const RAcc st = racc_unpack(seg_st[k][ch]);
      const int kq0 = min(ntot, k * per), kq1 = min(ntot, kq0 + per);
      seg_st[k][ch] = racc_pack(x);
      x = racc_combine(x, st, (float)(kq1 - kq0) * fL, w, u);
    }
  }
  __syncthreads();
  // 3. the state entering every chunk of the segment
  if (c >= p.C) return;
  RAcc x = racc_unpack(seg_st[sg][ch]);
  const size_t n_slots = (size_t)p.nch * p.B * p.NG * 64;  // (bounds-checked build)
  (void)n_slots;
  for (int q = q0; q < q1; ++q) {
    if (WKV_IN(p.hdr, bwd_slot(p, p.nch - 1 - q, b, c), n_slots)) p.rin[bwd_slot(p, p.nch - 1 - q, b, c)] = racc_pack(x);
    x = racc_combine(x, tot(q), fL, w, u);
  }
  if ((q0 < q1 && q1 == ntot) || (ntot == 0 && sg == 0)) p.rin[bwd_slot(p, 0, b, c)] = racc_pack(x);
}

// R2. One 32-thread CTA per (batch row, chunk, 32 channels), the chunk's k, v
// and g in shared memory (TMA). Forward replay of the chunk from x0[j]
// keeping the state at every 4th token (a checkpoint, in registers), then the
// tokens in reverse in groups of 4: the group's four states are recomputed
// from its checkpoint, and each token, from the last, gives dk, dv and its
// du, dw terms, then joins the reverse accumulator.
template <typename KV, int L>
__global__ void __launch_bounds__(32)
    wkv_bwd_chunk(const BwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const __grid_constant__ CUtensorMap tmg) {
  constexpr int NGRP = L / 4;
  extern __shared__ __align__(1024) unsigned char smem[];
  const KV* ks = reinterpret_cast<const KV*>(smem);
  const KV* vs = ks + L * 32;
  const float* gs = reinterpret_cast<const float*>(vs + L * 32);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + bwd_tile_bytes<KV, L>());
  const int lane = threadIdx.x;
  const int ngw = (p.C + 31) / 32;
  const long long item = blockIdx.x;
  const int gw = (int)(item % ngw);
  const int j = (int)((item / ngw) % p.nch);
  const int b = (int)(item / ((long long)ngw * p.nch));
  const int t0 = j * L;
  if (!bwd_load_tile<KV, L>(p, &tmk, &tmv, &tmg, smem, bar, gw, t0, b)) return;
  const int c = gw * 32 + lane;
  const unsigned vm = __ballot_sync(0xffffffffu, c < p.C);  // the lanes that go on (votes below)
  if (c >= p.C) return;
  const float w = __ldg(p.w + c), u = __ldg(p.u + c);
  const int n = min(L, p.T - t0);
  const size_t row0 = ((size_t)b * p.T + t0) * p.C + c;
  const size_t C = (size_t)p.C;
  if (!WKV_IN(p.hdr, (size_t)b * p.T + t0 + n - 1, (size_t)p.B * p.T) ||
      !WKV_IN(p.hdr, ((size_t)j * p.B + b) * p.C + c, (size_t)p.nch * p.B * p.C))
    return;
  auto kat = [&](int t) { return Elem<KV>::to_f32(ks[t * 32 + lane]); };
  auto vat = [&](int t) { return Elem<KV>::to_f32(vs[t * 32 + lane]); };

  // ---- forward replay with a checkpoint every 4 tokens
  Acc ck[NGRP];
  Acc s = acc_unpack(p.x0[bwd_slot(p, j, b, c)]);
#pragma unroll
  for (int gi = 0; gi < NGRP; ++gi) {
    ck[gi] = s;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int t = gi * 4 + q;
      if (t < n) add_token(s, kat(t), vat(t), w);
    }
  }

  // ---- reverse
  RAcc r = racc_unpack(p.rin[bwd_slot(p, j, b, c)]);  // at the chunk's end
  float du = 0.f, dw = 0.f;
#pragma unroll
  for (int gi = NGRP - 1; gi >= 0; --gi) {
    if (gi * 4 >= n) continue;
    Acc st[4];
    float kk[4], vv[4], gg[4];
    Acc x = ck[gi];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int t = gi * 4 + q;
      st[q] = x;
      if (t < n) {
        kk[q] = kat(t);
        vv[q] = vat(t);
        gg[q] = gs[t * 32 + lane];
        add_token(x, kk[q], vv[q], w);
      }
    }
#pragma unroll
    for (int q = 3; q >= 0; --q) {
      const int t = gi * 4 + q;
      if (t >= n) continue;
      const OutStat o = out_stat<true>(st[q], kk[q], vv[q], u, w, vm);
      const float rz = rcp(o.z);
      const float pp = gg[q] * rz, qq = -gg[q] * o.out * rz;
      // the reverse accumulator stands at t+1: Q = -qk - qu u + qc w
      // e^{k_t + Q}, exact where the exponent is large in some lane
      const float x1 = fmaf(r.qc, w, (kk[q] - r.qk) - r.qu * u);
      const float E1 = __any_sync(vm, fabsf(x1) > kExactFrom) ? exp_exact(r.qc, w, kk[q], r.qk, -r.qu * u)
                                                                : ex2(x1 * kLog2e);
      // (dw sums these over all tokens; its largest terms have exponents near
      // zero, so the rounded exponent suffices)
      const float E2 = ex2(fmaf(r.qc - st[q].nf - 1.f, w, (st[q].ma - r.qk) - r.qu * u) * kLog2e);  // e^{m_t + Q - w}
      const float pb = pp * o.b;
      p.dv[row0 + t * C] = fmaf(r.rn, E1, pb);
      p.dk[row0 + t * C] = fmaf(E1, fmaf(vv[q], r.rn, r.rd), pb * (vv[q] - o.out));
      du = fmaf(pb, vv[q] - o.out, du);
      dw = fmaf(-E2, fmaf(st[q].num, r.rn, st[q].den * r.rd), dw);
      // move the accumulator to position t and add token t
      r.qc -= 1.f;
      racc_add(r, o.key, o.uf, o.cnt, pp, qq, w, u);
    }
  }
  const size_t pi = ((size_t)j * p.B + b) * p.C + c;
  p.pdu[pi] = du;
  p.pdw[pi] = dw;
  if (j == 0 && p.d_num) {
    // the state passed in: dN_0 = rn e^{Q}, dD_0 = rd e^{Q}
    const size_t si = (size_t)b * p.C + c;
    float gn = 0.f, gd = 0.f, gm = 0.f;
    if (p.s_num) {
      const float num0 = p.s_num[si], den0 = p.s_den[si], m0 = p.s_max[si];
      if (den0 > 0.f && m0 > kNegBig) {
        const float f = exp_exact(r.qc, w, m0, r.qk, -r.qu * u);  // e^{m0 + Q}
        gn = r.rn * f;
        gd = r.rd * f;
        gm = fmaf(num0, gn, den0 * gd);
      }
    }
    p.d_num[si] = gn;
    p.d_den[si] = gd;
    p.d_max[si] = gm;
  }
}

// RED. du[c], dw[c] from the partials over (chunk, batch row): one warp per
// channel, lane l summing partials l, l+32, ... with compensation
// (Kahan-Babuska), then a fixed shuffle tree: the order depends on the shape
// only.
__global__ void __launch_bounds__(256) wkv_bwd_reduce(const BwdParams p) {
  // a warp per channel; lane l sums the partials of rows l, l + 32, ...
  // (four rows in flight per round), then a fixed shuffle tree
  const int lane = threadIdx.x & 31;
  const long long c = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (c >= p.C) return;
  float su = 0.f, cu = 0.f, sw = 0.f, cw = 0.f;
  const long long n = (long long)p.nch * p.B;
  for (long long i0 = lane; i0 < n; i0 += 4 * 32) {
    float xu[4], xw[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const long long i = i0 + r * 32;
      xu[r] = i < n ? p.pdu[i * p.C + c] : 0.f;
      xw[r] = i < n ? p.pdw[i * p.C + c] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float h, e;
      two_sum(su, xu[r], h, e);
      su = h;
      cu += e;
      two_sum(sw, xw[r], h, e);
      sw = h;
      cw += e;
    }
  }
  su += cu;
  sw += cw;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    su += __shfl_xor_sync(0xffffffffu, su, o);
    sw += __shfl_xor_sync(0xffffffffu, sw, o);
  }
  if (lane == 0) {
    p.du[c] = su;
    p.dw[c] = sw;
  }
}

}  // namespace wkv
