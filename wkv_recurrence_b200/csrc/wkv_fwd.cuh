// Forward kernels of the WKV operator over [B, T, C] sequences.
//
// All kernels run the recurrence of "Linear attention without writing a CUDA
// kernel", section "The recurrence", in the anchored form of wkv_device.cuh,
// one channel per register lane, VEC adjacent channels per thread, and stream
// k and v through shared memory with TMA (3-D tiled bulk copies of a
// [tokens x channel-group] box, completion on an mbarrier), or with plain
// loads where TMA cannot address the rows. The chunked scans come in three
// forms: in one launch with look-back between CTAs (wkv_fwd_chunk), in three
// launches with no waiting (wkv_tile_totals, wkv_tile_scan, then wkv_fwd_seq
// in chunked mode)
// and in persistent pipelined CTAs (wkv_fwd_pipe).
//
// * wkv_fwd_seq: one CTA per (batch row, channel group), walking all T tokens
//   through a STAGES-deep ring of [LT x CG] tiles. For many channels (B*C
//   large): the state never leaves registers.
//
// * wkv_fwd_chunk: for few channels and long T. T is cut into chunks of
//   L = NW*J tokens; a tile is (chunk, batch row, 64-channel group) and one
//   CTA of NW warps. Tiles are handed out in order by a ticket counter, so
//   every tile a CTA waits for belongs to a CTA that is already running. Per
//   tile, each warp loads its J tokens straight into registers and
//     1. folds them from the empty state into an aggregate (two passes: the
//        largest end-of-span exponent, then the weighted sums);
//     2. combines the aggregates of the warps before it (its in-tile prefix);
//        the last warp forms the tile total, publishes it and gathers the
//        tile's incoming state by look-back;
//     3. replays its tokens from registers, from (incoming state + prefix).
//   The associative combine of two spans (a, then b of len_b tokens) decays a
//   across b and adds the two relative to the larger exponent
//   (wkv::combine). The pages only say the recurrence has a parallel
//   prefix-scan form; this combine follows from the equation: a token's
//   weight at the end of a span is its key minus w times the tokens after it.
//
//   Look-back is blocked to keep results bitwise reproducible: chunks are
//   grouped G at a time; the last chunk of each group publishes its inclusive
//   prefix, every chunk publishes its own total, and chunk j combines the
//   prefix of the previous group's last chunk with the totals of the chunks
//   of its own group before it (at most G-1 of them). The order of combines
//   therefore depends on the shape and G only, never on timing.
//
//   Every wait (mbarrier phases, look-back flags) is bounded by a global-timer
//   limit; on expiry the kernel sets a status bit in the workspace header and
//   carries on with what it has, so that nothing hangs.
#pragma once

#include "wkv_device.cuh"

namespace wkv {

struct FwdParams {
  int B, T, C;
  int NG;              // channel groups per batch row
  const void* k;       // used only by the non-TMA path
  const void* v;
  const float* w;
  const float* u;
  void* out;
  const float* s_num;  // state in (all NULL = empty)
  const float* s_den;
  const float* s_max;
  float* o_num;        // state out (all NULL = not written)
  float* o_den;
  float* o_max;
  WsHeader* hdr;
  uint64_t timeout_ns;
  int vec_store;       // out rows allow VEC-wide stores
  // chunked kernel only
  int nch;             // chunks per sequence
  int G;               // look-back group
  int n_tiles;
  int inject_tile;     // tile that skips publishing (tests), -1 = none
  uint32_t* flags_a;   // [n_tiles]
  uint32_t* flags_p;   // [nblk * B * NG]
  float4* agg_a;       // [n_tiles][CG]
  float4* agg_p;       // [nblk * B * NG][CG] (single launch) or [n_tiles][NW][CG] (two launches)
  float4* x0;          // incoming states of chunks (three-launch scan)
  int chunk_len;       // chunked scans: tokens per chunk
  int stages;          // pipelined chunk scan: shared-memory stages in the ring
  int replay_chunks;   // three-launch scan: consecutive chunks per replay CTA
  int cluster;         // cluster kernel: CTAs per cluster
  int nseg;            // cluster kernel: segments per (batch row, 32-channel group)
  const float* w_t;    // per-token decay [B, T, C] in place of w, or NULL
  const void* r;       // receptance [B, T, C] (element type of k, v): out = sigmoid(r) wkv; or NULL
  float* wtot;         // three-launch scan with w_t: decay sum of each chunk total, [nch-1][B * NG][64]
};

// Programmatic dependent launch: let the next launch on the stream be
// scheduled, and wait for the launches before this one to finish (and their
// writes to be visible).
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// State in for one channel, anchored; empty when no state is passed.
__device__ __forceinline__ Acc state_in_acc(const FwdParams& p, int b, int c) {
  if (!p.s_num || c >= p.C) return acc_empty();
  const size_t i = (size_t)b * p.C + c;
  return acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
}

template <typename OUT, int VEC>
__device__ __forceinline__ void store_out(OUT* row, int c0, int C, bool vec_ok, const float (&o)[VEC]) {
  if constexpr (VEC == 1) {
    // one channel per thread: callers store only for c0 < C
    row[c0] = Elem<OUT>::from_f32(o[0]);
  } else if (vec_ok && c0 + VEC <= C) {
    store_vec<OUT, VEC>(row + c0, o);
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e)
      if (c0 + e < C) row[c0 + e] = Elem<OUT>::from_f32(o[e]);
  }
}

// A compile-time flag passed to generic lambdas (so that one body is compiled
// once per value).
template <bool V>
struct Flag {
  static constexpr bool value = V;
};

// The receptance gate on VEC outputs of one token row (out = sigmoid(r) wkv),
// when the call has one: r is [B, T, C] with the element type of k and v;
// `row` is the offset of (b, t, 0).
template <typename KV, int VEC>
__device__ __forceinline__ void gate_row(const FwdParams& p, size_t row, int c0, float (&o)[VEC]) {
  if (!p.r) return;
  const KV* rr = reinterpret_cast<const KV*>(p.r) + row;
#pragma unroll
  for (int e = 0; e < VEC; ++e)
    if (c0 + e < p.C) o[e] = gate(o[e], Elem<KV>::to_f32(rr[c0 + e]));
}

// Bytes of one shared-memory stage of the sequential kernel: LT tokens x CG
// channels of k and v, and of w_t with per-token decays.
template <typename KV, int LT, int CG, bool kWT>
__host__ __device__ constexpr uint32_t seq_stage_bytes() {
  return (uint32_t)(LT * CG * (2 * sizeof(KV) + (kWT ? sizeof(float) : 0)));
}

template <typename KV>
__device__ __forceinline__ void coop_load_tile(KV* dst, const KV* src, int b, int t0, int rows, int cbase, int CG,
                                               int T, int C) {
  // plain, masked copy of a [rows x CG] box (zero outside [0,T) x [0,C))
  for (int i = threadIdx.x; i < rows * CG; i += blockDim.x) {
    const int r = i / CG, cc = i % CG;
    const int t = t0 + r, c = cbase + cc;
    KV x = Elem<KV>::from_f32(0.f);
    if (t < T && c < C) x = src[((size_t)b * T + t) * C + c];
    dst[i] = x;
  }
}

// ---------------------------------------------------------------------------
// sequential-over-T kernel
// ---------------------------------------------------------------------------
// kChunked: the replay pass of the three-launch scan. A CTA then takes
// R = p.replay_chunks consecutive chunks (R * p.chunk_len tokens) of one batch
// row and starts from the incoming state of the first, which the scan pass
// wrote to p.x0 ([nch][B * NG][64] with p.NG 64-channel groups); the grid is
// B * ceil(nch / R) * ceil(C / CG), replays taken from the sequence's end
// (the chunks the totals pass read last are the ones still in L2). It issues
// its first copies (inputs only) before waiting (griddepcontrol.wait) for the
// scan, and only the CTA that ends the sequence writes the state out.
template <typename KV, typename OUT, int VEC, int THREADS, int LT, int STAGES, bool kTMA, bool kChunked,
          bool kWT>
__global__ void __launch_bounds__(THREADS)
    wkv_fwd_seq(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                const __grid_constant__ CUtensorMap tmw) {
  constexpr int CG = THREADS * VEC;
  constexpr int kTile = LT * CG;  // elements per tensor per stage
  constexpr uint32_t kStageBytes = seq_stage_bytes<KV, LT, CG, kWT>();
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  // stage s: k tile, v tile (KV), then the w_t tile (fp32)
  auto ktile = [&](int s) { return reinterpret_cast<KV*>(smem + (size_t)s * kStageBytes); };
  auto wtile = [&](int s) {
    return reinterpret_cast<float*>(smem + (size_t)s * kStageBytes + 2 * kTile * sizeof(KV));
  };

  const int tid = threadIdx.x;
  const int T = p.T, C = p.C;
  const int ngs = kChunked ? (C + CG - 1) / CG : p.NG;  // channel groups of this kernel
  const int bj = blockIdx.x / ngs;
  const int g = blockIdx.x % ngs;
  const int nseq = kChunked ? (p.nch + p.replay_chunks - 1) / p.replay_chunks : 1;  // replays per row
  // replays in reverse chunk order, batch rows inner: the totals pass read
  // the chunks in order, so the last ones it read are the ones still in L2
  const int b = kChunked ? bj % p.B : bj;
  const int js = kChunked ? nseq - 1 - bj / p.B : 0;  // replay
  const int jc = js * (kChunked ? p.replay_chunks : 1);  // its first chunk
  const int tbeg = kChunked ? jc * p.chunk_len : 0;
  const int tend = kChunked ? min(T, tbeg + p.replay_chunks * p.chunk_len) : T;
  const int c0 = g * CG + tid * VEC;
  const int ntile = (tend - tbeg + LT - 1) / LT;

  auto issue = [&](int s, int t) {
    mbar_arrive_expect_tx(&full[s], kStageBytes);
    tma_load_3d(ktile(s), &tmk, &full[s], g * CG, t, b);
    tma_load_3d(ktile(s) + kTile, &tmv, &full[s], g * CG, t, b);
    if (kWT) tma_load_3d(wtile(s), &tmw, &full[s], g * CG, t, b);
  };
  if (kTMA && tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    for (int s = 0; s < STAGES && s < ntile; ++s) issue(s, tbeg + s * LT);
  }

  float w[VEC], u[VEC], cb[VEC], lo[VEC];
  Acc st[VEC];
  bool fast = true;
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const int c = c0 + e;
    const bool ok = c < C;
    w[e] = (ok && !kWT) ? p.w[c] : 0.f;
    u[e] = ok ? p.u[c] : 0.f;
    lo[e] = 0.f;
    fast &= fast_uw(u[e], w[e]);
    cb[e] = ex2(fminf(fmaxf(u[e] - w[e], -kFastUW), kFastUW) * kLog2e);
    st[e] = acc_empty();
    if (!kChunked && ok && p.s_num) {
      const size_t i = (size_t)b * C + c;
      st[e] = acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
    }
  }
  if (kChunked) {
    grid_wait_prerequisites();  // the scan pass has written the incoming states
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const int c = c0 + e;
      const size_t xi = ((size_t)jc * p.B * p.NG + (size_t)b * p.NG + c / 64) * 64 + c % 64;
      if (c < C && WKV_IN(p.hdr, xi, (size_t)p.nch * p.B * p.NG * 64)) st[e] = acc_unpack(p.x0[xi]);
    }
  }
  fast = __all_sync(0xffffffffu, fast);  // one path per warp
  __syncthreads();

  OUT* out = reinterpret_cast<OUT*>(p.out);
  const bool vec_ok = p.vec_store != 0;
  int issued = (STAGES < ntile) ? STAGES : ntile;  // tiles whose loads were issued
  int aborted_at = -1;
  for (int i = 0; i < ntile; ++i) {
    const int s = kTMA ? (i % STAGES) : 0;
    const int t0 = tbeg + i * LT;
    if (kTMA) {
      const bool ok = mbar_wait(&full[s], (i / STAGES) & 1, p.timeout_ns);
      if (__syncthreads_or(!ok)) {
        aborted_at = i;
        break;
      }
    } else {
      coop_load_tile<KV>(ktile(0), reinterpret_cast<const KV*>(p.k), b, t0, LT, g * CG, CG, T, C);
      coop_load_tile<KV>(ktile(0) + kTile, reinterpret_cast<const KV*>(p.v), b, t0, LT, g * CG, CG, T, C);
      if (kWT) coop_load_tile<float>(wtile(0), p.w_t, b, t0, LT, g * CG, CG, T, C);
      __syncthreads();
    }
    const KV* ks = ktile(s) + tid * VEC;
    const KV* vs = ks + kTile;
    const float* wsm = wtile(s) + tid * VEC;
    const int nv = min(LT, tend - t0);
    OUT* orow = out + ((size_t)b * T + t0) * C;
    const size_t rrow = ((size_t)b * T + t0) * C;
    if (c0 < C && WKV_IN(p.hdr, (size_t)b * T + t0 + nv - 1, (size_t)p.B * T)) {
      if (kWT) {
        for (int j = 0; j < nv; ++j) {
          float kx[VEC], vx[VEC], wx[VEC], o[VEC];
          load_vec<KV, VEC>(ks + j * CG, kx);
          load_vec<KV, VEC>(vs + j * CG, vx);
          load_vec<float, VEC>(wsm + j * CG, wx);
#pragma unroll
          for (int e = 0; e < VEC; ++e) o[e] = step_token_wt(st[e], lo[e], kx[e], vx[e], wx[e], u[e]);
          gate_row<KV, VEC>(p, rrow + (size_t)j * C, c0, o);
          store_out<OUT, VEC>(orow + (size_t)j * C, c0, C, vec_ok, o);
        }
      } else if (nv == LT && fast) {
        // the tile's hot loop, compiled once with and once without the gate
        // (no per-token test of p.r)
        auto tile = [&](auto gated) {
          constexpr bool kGate = decltype(gated)::value;
          constexpr int NB = LT < 8 ? LT : 8;  // tokens per block of step_tokens
#pragma unroll
          for (int j0 = 0; j0 < LT; j0 += NB) {
            float kb[NB][VEC], vb[NB][VEC], ob[NB][VEC];
#pragma unroll
            for (int jj = 0; jj < NB; ++jj) {
              load_vec<KV, VEC>(ks + (j0 + jj) * CG, kb[jj]);
              load_vec<KV, VEC>(vs + (j0 + jj) * CG, vb[jj]);
            }
            step_tokens<NB, VEC>(st, kb, vb, w, cb, ob);
#pragma unroll
            for (int jj = 0; jj < NB; ++jj) {
              if (kGate) gate_row<KV, VEC>(p, rrow + (size_t)(j0 + jj) * C, c0, ob[jj]);
              store_out<OUT, VEC>(orow + (size_t)(j0 + jj) * C, c0, C, vec_ok, ob[jj]);
            }
          }
        };
        if (p.r) {
          tile(Flag<true>{});
        } else {
          tile(Flag<false>{});
        }
      } else if (nv == LT) {
#pragma unroll 4
        for (int j = 0; j < LT; ++j) {
          float kx[VEC], vx[VEC], o[VEC];
          load_vec<KV, VEC>(ks + j * CG, kx);
          load_vec<KV, VEC>(vs + j * CG, vx);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
            add_token(st[e], kx[e], vx[e], w[e]);
          }
          gate_row<KV, VEC>(p, rrow + (size_t)j * C, c0, o);
          store_out<OUT, VEC>(orow + (size_t)j * C, c0, C, vec_ok, o);
        }
      } else {
        for (int j = 0; j < nv; ++j) {
          float kx[VEC], vx[VEC], o[VEC];
          load_vec<KV, VEC>(ks + j * CG, kx);
          load_vec<KV, VEC>(vs + j * CG, vx);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
            add_token(st[e], kx[e], vx[e], w[e]);
          }
          gate_row<KV, VEC>(p, rrow + (size_t)j * C, c0, o);
          store_out<OUT, VEC>(orow + (size_t)j * C, c0, C, vec_ok, o);
        }
      }
    }
    __syncthreads();  // every thread is done with stage s
    if (kTMA && tid == 0 && i + STAGES < ntile) {
      fence_proxy_async_smem();
      issue(s, tbeg + (i + STAGES) * LT);
      ++issued;
    }
  }

  if (aborted_at >= 0) {
    if (tid == 0) {
      atomicOr(&p.hdr->status, kStatusWaitTimeout);
      // copies still in flight (tiles aborted_at .. issued-1): give each a
      // bounded chance to land before the CTA leaves
      for (int x = aborted_at; x < issued; ++x) (void)mbar_wait(&full[x % STAGES], (x / STAGES) & 1, p.timeout_ns);
    }
    return;
  }

  if (p.o_num && c0 < C && (!kChunked || js == nseq - 1)) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const int c = c0 + e;
      const size_t i = (size_t)b * C + c;
      if (c < C && WKV_IN(p.hdr, i, (size_t)p.B * C)) {
        p.o_num[i] = st[e].num;
        p.o_den[i] = st[e].den;
        p.o_max[i] = kWT ? acc_max_e_wt(st[e], lo[e]) : acc_max_e(st[e], w[e]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// chunked-scan kernel
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* q) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(q) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void named_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(N) : "memory");
}

// Named barrier that also ORs a predicate over the N participating threads.
template <int N>
__device__ __forceinline__ bool named_sync_or(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "n"(N)
      : "memory");
  return r != 0;
}

// Aggregate of one warp's span of n <= J tokens from the empty state, read
// from a shared-memory tile in two passes: first the largest exponent M that
// any token has at the end of the span (s_i = k_i - (n-1-i) w, one fma each),
// then the sums of e^{s_i - M} v_i and e^{s_i - M}. No per-token
// compare-and-select is needed. The result is anchored at M with count 0.
// `ks`, `vs` point at this lane's channels in the span's first row; rows are
// CG elements apart.
template <typename KV, int J, int VEC, int CG>
__device__ __forceinline__ void aggregate_tile_span(const KV* ks, const KV* vs, int n, const float (&w)[VEC],
                                                    Acc (&agg)[VEC]) {
  float M[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) M[e] = kNegBig;
  const float last = (float)(n - 1);
#pragma unroll
  for (int i = 0; i < J; ++i) {
    if (i < n) {
      float kx[VEC];
      load_vec<KV, VEC>(ks + i * CG, kx);
#pragma unroll
      for (int e = 0; e < VEC; ++e) M[e] = fmaxf(M[e], fmaf((float)i - last, w[e], kx[e]));
    }
  }
  float ML[VEC], num[VEC], den[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    ML[e] = M[e] * kLog2e;
    num[e] = den[e] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < J; ++i) {
    if (i < n) {
      float kx[VEC], vx[VEC];
      load_vec<KV, VEC>(ks + i * CG, kx);
      load_vec<KV, VEC>(vs + i * CG, vx);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float x = ex2(fmaf(fmaf((float)i - last, w[e], kx[e]), kLog2e, -ML[e]));
        num[e] = fmaf(x, vx[e], num[e]);
        den[e] += x;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    if (n <= 0) {
      agg[e] = acc_empty();
    } else {
      // all weights share the factor 2^{M log2e - ML} from rounding ML
      const float corr = fmaf(M[e], kLog2e, -ML[e]);
      const float fix = fmaf(-corr, 0.6931471805599453f, 1.f);
      agg[e] = Acc{num[e] * fix, den[e] * fix, M[e], 0.f};
    }
  }
}

// Aggregate of one span of n <= J tokens with per-token decays ("RWKV-v6
// Architecture", section "2. Dynamic Data-Dependent Decay"), anchored at the
// span's end: token i has exponent s_i = k_i - (w_{i+1} + ... + w_{n-1})
// there. The suffix sums are compensated (two_sum). Also returns the span's
// decay sum (what the span does to everything before it). `ws` points at this
// lane's channels of the span's w_t rows, CG apart like k and v.
template <typename KV, int J, int VEC, int CG>
__device__ __forceinline__ void aggregate_span_wt(const KV* ks, const KV* vs, const float* ws, int n,
                                                  Acc (&agg)[VEC], float (&wsum)[VEC]) {
  float sx[J][VEC];
  float hi[VEC], lo[VEC], M[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    hi[e] = lo[e] = 0.f;
    M[e] = kNegBig;
  }
#pragma unroll
  for (int i = J - 1; i >= 0; --i) {
    if (i < n) {
      float kx[VEC], wx[VEC];
      load_vec<KV, VEC>(ks + i * CG, kx);
      load_vec<float, VEC>(ws + i * CG, wx);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        sx[i][e] = (kx[e] - hi[e]) - lo[e];
        M[e] = fmaxf(M[e], sx[i][e]);
        float h, er;
        two_sum(hi[e], wx[e], h, er);
        hi[e] = h;
        lo[e] += er;
      }
    }
  }
  float ML[VEC], num[VEC], den[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    ML[e] = M[e] * kLog2e;
    num[e] = den[e] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < J; ++i) {
    if (i < n) {
      float vx[VEC];
      load_vec<KV, VEC>(vs + i * CG, vx);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float x = ex2(fmaf(sx[i][e], kLog2e, -ML[e]));
        num[e] = fmaf(x, vx[e], num[e]);
        den[e] += x;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    wsum[e] = hi[e] + lo[e];
    if (n <= 0) {
      agg[e] = acc_empty();
    } else {
      const float corr = fmaf(M[e], kLog2e, -ML[e]);
      const float fix = fmaf(-corr, 0.6931471805599453f, 1.f);
      agg[e] = Acc{num[e] * fix, den[e] * fix, M[e], 0.f};
    }
  }
}

// Incoming state of chunk j from the published values of its look-back group
// (chunks first .. j-1) and, when given, the previous group's inclusive prefix:
// x = prefix, then combined with each chunk total in chunk order (the order
// of combines is fixed, so results do not depend on timing). Loading several
// totals before combining them (kBatch > 1) was measured: it costs registers
// (and so resident CTAs) and gained nothing, so they are loaded one by one.
template <int VEC, int CG, int L>
__device__ __forceinline__ void gather_group(const FwdParams& p, Acc (&x)[VEC], int first, int j, int bg, int cl,
                                             const float (&w)[VEC], bool has_prefix, int qb) {
  constexpr int kBatch = 1;
  const int BNG = p.B * p.NG;
  if (has_prefix) {
    const float4* src = p.agg_p + ((size_t)(qb - 1) * BNG + bg) * CG + cl;
#pragma unroll
    for (int e = 0; e < VEC; ++e) x[e] = acc_unpack(ld_relaxed_f4(src + e));
  }
  for (int j0 = first; j0 < j; j0 += kBatch) {
    float4 t[kBatch][VEC];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (j0 + i < j) {
        const float4* src = p.agg_a + ((size_t)(j0 + i) * BNG + bg) * CG + cl;
#pragma unroll
        for (int e = 0; e < VEC; ++e) t[i][e] = ld_relaxed_f4(src + e);
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (j0 + i < j) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[e] = combine(x[e], acc_unpack(t[i][e]), (float)L, w[e]);
      }
    }
  }
}

// Tile = 64 channels (32 lanes x 2) by L = NW * J tokens of one batch row, one
// CTA of NW compute warps plus one scan warp. Thread 0 takes the tile's ticket
// and starts its TMA copy (k and v boxes into shared memory); meanwhile the
// scan warp gathers the tile's incoming state from earlier chunks (look-back),
// which needs nothing from this tile. Compute warp wp owns tokens
// [t0 + wp*J, t0 + (wp+1)*J): it folds them into an aggregate, takes the
// aggregates of the compute warps before it as its in-tile prefix, and the last
// compute warp publishes the tile total -- before waiting for the scan warp,
// so that no tile's total waits on another tile's look-back. Then every
// compute warp replays its tokens from shared memory.
template <typename KV, typename OUT, int NW, int J, bool kTMA>
__global__ void __launch_bounds__((NW + 1) * 32)
    wkv_fwd_chunk(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  constexpr int VEC = 2;
  constexpr int CG = 32 * VEC;
  constexpr int L = NW * J;
  constexpr int kTile = L * CG;
  constexpr uint32_t kBytes = 2u * kTile * sizeof(KV);
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* ktile = reinterpret_cast<KV*>(smem);
  KV* vtile = ktile + kTile;
  float4* sh_agg = reinterpret_cast<float4*>(smem + kBytes);  // [NW][CG]
  float4* sh_x = sh_agg + NW * CG;                             // [CG]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sh_x + CG);
  int* sh_tile = reinterpret_cast<int*>(bar + 1);

  const int lane = threadIdx.x & 31;
  const int wp = threadIdx.x >> 5;
  const bool scan = (wp == NW);
  const int T = p.T, C = p.C;
  const int BNG = p.B * p.NG;
  const uint32_t target = *reinterpret_cast<volatile uint32_t*>(&p.hdr->epoch) + 1u;

  if (threadIdx.x == 0) {
    const int t = (int)atomicAdd(&p.hdr->ticket, 1u);
    *sh_tile = t;
    if (kTMA) {
      const int jj = t / BNG, bgg = t % BNG;
      mbar_init(bar, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(bar, kBytes);
      tma_load_3d(ktile, &tmk, bar, (bgg % p.NG) * CG, jj * L, bgg / p.NG);
      tma_load_3d(vtile, &tmv, bar, (bgg % p.NG) * CG, jj * L, bgg / p.NG);
    }
  }
  __syncthreads();
  const int tile = *sh_tile;
  const int j = tile / BNG;
  const int bg = tile % BNG;
  const int b = bg / p.NG, g = bg % p.NG;
  const int t0 = j * L;
  const int cl = lane * VEC;
  const int c0 = g * CG + cl;
  const bool last_chunk = (j == p.nch - 1);
  const bool inject = (tile == p.inject_tile);
  float w[VEC], u[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const bool ok = c0 + e < C;
    w[e] = ok ? __ldg(p.w + c0 + e) : 0.f;
    u[e] = ok ? __ldg(p.u + c0 + e) : 0.f;
  }

  if (scan) {
    // ---- hand the workspace back for the next launch: the CTA that counts
    // itself last resets the ticket counter and advances the epoch. Every CTA
    // counts itself only after reading the epoch and taking its ticket (both
    // before the __syncthreads above), and neither is read again during the
    // launch, so this can happen at the start instead of at the end, off the
    // tile's path. The next launch on the stream starts after this one ends.
    if (lane == 0) {
      const uint32_t prev = atomicAdd(&p.hdr->done, 1u);
      if (prev == (uint32_t)p.n_tiles - 1u) {
        p.hdr->ticket = 0;
        p.hdr->done = 0;
        __threadfence();
        atomicExch(&p.hdr->epoch, target);
      }
    }
    // ---- look-back: incoming state of the tile (overlaps the TMA copy)
    Acc x[VEC];
    const int qb = j / p.G;
    const int first = qb * p.G;
    // Only chunk 0 reads the state in; its published total already contains
    // it, so no later tile reads the caller's state (which state_out may alias).
#pragma unroll
    for (int e = 0; e < VEC; ++e) x[e] = (j == 0) ? state_in_acc(p, b, c0 + e) : acc_empty();
    if (j > 0) {
      const uint32_t* fp = p.flags_p + (size_t)(qb - 1) * BNG + bg;
      bool ready = false;
      uint64_t tstart = 0;
      while (true) {
        bool all = (qb == 0) || ld_relaxed_u32(fp) == target;
        for (int jj = first + lane; jj < j; jj += 32)
          all &= ld_relaxed_u32(p.flags_a + (size_t)jj * BNG + bg) == target;
        all = __all_sync(0xffffffffu, all);
        if (all) {
          ready = true;
          break;
        }
        if (tstart == 0) {
          tstart = global_ns();
        } else if (global_ns() - tstart > p.timeout_ns) {
          break;
        }
        __nanosleep(32);
      }
      if (!ready && lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
      fence_acq_rel_gpu();
      gather_group<VEC, CG, L>(p, x, first, j, bg, cl, w, qb > 0, qb);
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) sh_x[cl + e] = acc_pack(x[e]);
    named_sync<(NW + 1) * 32>(2);  // (A) incoming state ready; totals published
  } else {
    // ---- compute warps
    const int ts = t0 + wp * J;
    const int nv = max(0, min(J, T - ts));
    const int p_last = last_chunk ? (T - 1 - t0) / J : NW - 1;
    bool copy_ok = true;
    if (kTMA) {
      copy_ok = mbar_wait(bar, 0, p.timeout_ns);
      if (!copy_ok && lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
    } else {
      for (int i = threadIdx.x; i < kTile; i += NW * 32) {
        const int r = i / CG, cc = i % CG;
        const int t = t0 + r, c = g * CG + cc;
        KV kk = Elem<KV>::from_f32(0.f), vv = Elem<KV>::from_f32(0.f);
        if (t < T && c < C) {
          kk = reinterpret_cast<const KV*>(p.k)[((size_t)b * T + t) * C + c];
          vv = reinterpret_cast<const KV*>(p.v)[((size_t)b * T + t) * C + c];
        }
        ktile[i] = kk;
        vtile[i] = vv;
      }
      named_sync<NW * 32>(1);
    }
    const KV* ks = ktile + (wp * J) * CG + cl;
    const KV* vs = vtile + (wp * J) * CG + cl;
    // 1. aggregate of this warp's span
    {
      Acc agg[VEC];
      if (last_chunk && wp >= p_last) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) agg[e] = acc_empty();
      } else {
        aggregate_tile_span<KV, J, VEC, CG>(ks, vs, nv, w, agg);
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) sh_agg[wp * CG + cl + e] = acc_pack(agg[e]);
    }
    named_sync<NW * 32>(1);
    // 2. in-tile prefix; the last compute warp publishes the tile total
    Acc pre[VEC], tot[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) pre[e] = acc_empty();
    for (int q = 0; q < wp; ++q) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) pre[e] = combine(pre[e], acc_unpack(sh_agg[q * CG + cl + e]), (float)J, w[e]);
    }
    if (wp == NW - 1) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) tot[e] = combine(pre[e], acc_unpack(sh_agg[wp * CG + cl + e]), (float)nv, w[e]);
      if (!last_chunk && WKV_IN(p.hdr, (size_t)tile * CG + cl + VEC - 1, (size_t)p.n_tiles * CG)) {
        float4* dst = p.agg_a + (size_t)tile * CG + cl;
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          dst[e] = acc_pack(j == 0 ? combine(state_in_acc(p, b, c0 + e), tot[e], (float)L, w[e]) : tot[e]);
        __threadfence();
        __syncwarp();
        if (lane == 0 && !inject) st_release_u32(p.flags_a + tile, target);
      }
    }
    named_sync<(NW + 1) * 32>(2);  // (A) incoming state ready
    if (wp == NW - 1 && !last_chunk && (j % p.G) == p.G - 1) {
      // the last chunk of a look-back group publishes its inclusive prefix
      const int qb = j / p.G;
      float4* dst = p.agg_p + ((size_t)qb * BNG + bg) * CG + cl;
#pragma unroll
      for (int e = 0; e < VEC; ++e) dst[e] = acc_pack(combine(acc_unpack(sh_x[cl + e]), tot[e], (float)L, w[e]));
      __threadfence();
      __syncwarp();
      if (lane == 0 && !inject) st_release_u32(p.flags_p + (size_t)qb * BNG + bg, target);
    }
    // 3. replay this warp's tokens from shared memory
    if (nv > 0 && copy_ok && WKV_IN(p.hdr, (size_t)b * T + ts + nv - 1, (size_t)p.B * T)) {
      float cb[VEC];
      bool fast = true;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        fast &= fast_uw(u[e], w[e]);
        cb[e] = ex2(fminf(fmaxf(u[e] - w[e], -kFastUW), kFastUW) * kLog2e);
      }
      fast = __all_sync(0xffffffffu, fast);
      Acc st[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) st[e] = combine(acc_unpack(sh_x[cl + e]), pre[e], (float)(wp * J), w[e]);
      OUT* orow = reinterpret_cast<OUT*>(p.out) + ((size_t)b * T + ts) * C + c0;
      const bool lane_vec = p.vec_store != 0 && c0 + VEC <= C;
      if (fast && nv == J) {
        constexpr int NB = J < 8 ? J : 8;  // tokens per block of step_tokens
#pragma unroll
        for (int i0 = 0; i0 < J; i0 += NB) {
          float kb[NB][VEC], vb[NB][VEC], ob[NB][VEC];
#pragma unroll
          for (int ii = 0; ii < NB; ++ii) {
            load_vec<KV, VEC>(ks + (i0 + ii) * CG, kb[ii]);
            load_vec<KV, VEC>(vs + (i0 + ii) * CG, vb[ii]);
          }
          step_tokens<NB, VEC>(st, kb, vb, w, cb, ob);
#pragma unroll
          for (int ii = 0; ii < NB; ++ii) {
            gate_row<KV, VEC>(p, ((size_t)b * T + ts + i0 + ii) * C, c0, ob[ii]);
            if (lane_vec) {
              stg_stream<OUT, VEC>(orow + (size_t)(i0 + ii) * C, ob[ii]);
            } else {
#pragma unroll
              for (int e = 0; e < VEC; ++e)
                if (c0 + e < C) orow[(size_t)(i0 + ii) * C + e] = Elem<OUT>::from_f32(ob[ii][e]);
            }
          }
        }
      } else if (fast) {
        for (int i = 0; i < nv; ++i) {
          float kx[VEC], vx[VEC], o[VEC];
          load_vec<KV, VEC>(ks + i * CG, kx);
          load_vec<KV, VEC>(vs + i * CG, vx);
#pragma unroll
          for (int e = 0; e < VEC; ++e) o[e] = step_token(st[e], kx[e], vx[e], w[e], cb[e]);
          gate_row<KV, VEC>(p, ((size_t)b * T + ts + i) * C, c0, o);
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if (c0 + e < C) orow[(size_t)i * C + e] = Elem<OUT>::from_f32(o[e]);
        }
      } else {
        for (int i = 0; i < nv; ++i) {
          float kx[VEC], vx[VEC], o[VEC];
          load_vec<KV, VEC>(ks + i * CG, kx);
          load_vec<KV, VEC>(vs + i * CG, vx);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
            add_token(st[e], kx[e], vx[e], w[e]);
          }
          gate_row<KV, VEC>(p, ((size_t)b * T + ts + i) * C, c0, o);
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if (c0 + e < C) orow[(size_t)i * C + e] = Elem<OUT>::from_f32(o[e]);
        }
      }
      if (last_chunk && wp == p_last && p.o_num) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          if (c0 + e < C) {
            const size_t i = (size_t)b * C + c0 + e;
            p.o_num[i] = st[e].num;
            p.o_den[i] = st[e].den;
            p.o_max[i] = acc_max_e(st[e], w[e]);
          }
        }
      }
    }
    if (kTMA && !copy_ok && threadIdx.x == 0) (void)mbar_wait(bar, 0, p.timeout_ns);  // bounded drain
  }

}

// ---------------------------------------------------------------------------
// chunked scan in three launches: chunk totals, their scan, the replay
// ---------------------------------------------------------------------------
//
// The tiles of wkv_fwd_chunk (64 channels x L = NW * J tokens, one CTA each),
// with the look-back replaced by a launch boundary, so that no CTA ever waits
// for another:
//   A (wkv_tile_totals): every tile but those of the last chunk is copied in
//     (TMA), folded from the empty state into its total, and the total is
//     written to the workspace;
//   S (wkv_tile_scan): for each (batch row, channel), the incoming state of
//     every chunk: the state in combined with the totals of the chunks before
//     it, as a two-level scan (segments of chunks, then within segments);
//   B (wkv_fwd_seq in chunked mode): every (batch row, chunk) is replayed as
//     an independent sequence of chunk_len tokens from its incoming state, one
//     channel per thread, streaming k and v again through TMA stages.
// k and v are read twice from memory: for inputs that fit in L2 the second
// read hits L2. A is an ordinary launch; S (behind A) and B are launched with
// programmatic stream serialization, so that each may be resident before the
// one ahead of it ends:
//   A lets S be scheduled once its copies are issued;
//   S reads w, then waits (griddepcontrol.wait) for A before its first total;
//   B issues its first copies (inputs only) while S runs and waits for S
//     before reading an incoming state.
// Both are scheduled only after A has started, so every read of the call's
// inputs follows the end of the launch ahead of the call. Only S reads the
// caller's state in, and it completes before B writes the state out (from
// the last chunk), so the two may alias. The order of combines depends on the
// shape only.

__device__ __forceinline__ float4 ldg_f4(const float4* q) {
  float4 r;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(q));
  return r;
}

// Pass A. Grid: (nch - 1) * B * NG CTAs of NW warps; tile = blockIdx.x in
// chunk-major order. Every tile here is a full chunk (the last chunk, which
// alone can be partial, has no total to compute).
template <typename KV, int NW, int J, bool kWT>
__global__ void __launch_bounds__(NW * 32)
    wkv_tile_totals(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmw) {
  constexpr int VEC = 2;
  constexpr int CG = 32 * VEC;
  constexpr int L = NW * J;
  constexpr int kTile = L * CG;
  constexpr uint32_t kBytes = (uint32_t)(2u * kTile * sizeof(KV) + (kWT ? kTile * sizeof(float) : 0));
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* ktile = reinterpret_cast<KV*>(smem);
  float* wtile = reinterpret_cast<float*>(smem + 2u * kTile * sizeof(KV));  // (kWT)
  float4* sh_agg = reinterpret_cast<float4*>(smem + kBytes);  // [NW][CG]
  float* sh_w = reinterpret_cast<float*>(sh_agg + NW * CG);   // [NW][CG] (kWT)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sh_w + (kWT ? NW * CG : 0));

  const int lane = threadIdx.x & 31;
  const int wp = threadIdx.x >> 5;
  const int BNG = p.B * p.NG;
  const int tile = blockIdx.x;
  const int j = tile / BNG, bg = tile % BNG;
  const int cl = lane * VEC;
  const int c0 = (bg % p.NG) * CG + cl;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, kBytes);
    tma_load_3d(ktile, &tmk, bar, (bg % p.NG) * CG, j * L, bg / p.NG);
    tma_load_3d(ktile + kTile, &tmv, bar, (bg % p.NG) * CG, j * L, bg / p.NG);
    if (kWT) tma_load_3d(wtile, &tmw, bar, (bg % p.NG) * CG, j * L, bg / p.NG);
  }
  grid_launch_dependents();  // the scan may be scheduled (it waits for this grid)
  __syncthreads();
  float w[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) w[e] = (!kWT && c0 + e < p.C) ? __ldg(p.w + c0 + e) : 0.f;
  const bool ok = mbar_wait(bar, 0, p.timeout_ns);
  Acc a[VEC];
  float ws[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) ws[e] = 0.f;
  if (ok) {
    const int o = (wp * J) * CG + cl;
    if (kWT) {
      aggregate_span_wt<KV, J, VEC, CG>(ktile + o, ktile + kTile + o, wtile + o, J, a, ws);
    } else {
      aggregate_tile_span<KV, J, VEC, CG>(ktile + o, ktile + kTile + o, J, w, a);
    }
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e) a[e] = acc_empty();
    if (lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    sh_agg[wp * CG + cl + e] = acc_pack(a[e]);
    if (kWT) sh_w[wp * CG + cl + e] = ws[e];
  }
  __syncthreads();
  if (wp == 0) {
    Acc t[VEC];
    float wt[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      t[e] = acc_unpack(sh_agg[cl + e]);
      wt[e] = kWT ? sh_w[cl + e] : 0.f;
    }
    for (int q = 1; q < NW; ++q) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        if (kWT) {
          const float wq = sh_w[q * CG + cl + e];
          t[e] = combine_wt(t[e], acc_unpack(sh_agg[q * CG + cl + e]), wq);
          wt[e] += wq;
        } else {
          t[e] = combine(t[e], acc_unpack(sh_agg[q * CG + cl + e]), (float)J, w[e]);
        }
      }
    }
    float4* dst = p.agg_a + (size_t)tile * CG + cl;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      if (!WKV_IN(p.hdr, (size_t)tile * CG + cl + e, (size_t)(p.nch - 1) * BNG * CG)) continue;
      dst[e] = acc_pack(t[e]);
      if (kWT) p.wtot[(size_t)tile * CG + cl + e] = wt[e];
    }
  }
  if (!ok && threadIdx.x == 0) (void)mbar_wait(bar, 0, p.timeout_ns);  // bounded drain
}

// Pass S. Grid: B * NG * 4 CTAs of 16 * SEG threads: a CTA takes 16 of the
// 64 channels of a (batch row, channel group), and SEG threads per channel
// each own a contiguous segment of the nch - 1 chunk totals: (1) each
// segment's total; (2) one thread per channel walks the segment totals once,
// from the state in, leaving each segment's incoming state in shared memory;
// (3) each thread walks its segment again, writing each chunk's incoming
// state to p.x0 [nch][B * NG][64] (and the last chunk's). Behind the totals
// pass it is launched with programmatic stream serialization and waits
// (griddepcontrol.wait) for that pass before its first load of a total. The totals are read-only from then on,
// so they are loaded through the non-coherent path, eight at a time; a
// segment of at most eight is loaded once and kept in registers.
template <int SEG, bool kWT>
__global__ void __launch_bounds__(16 * SEG) wkv_tile_scan(const FwdParams p, int L) {
  constexpr int CG = 64, CH = 16;
  __shared__ float4 seg_st[SEG][CH];
  __shared__ float seg_w[SEG][CH];  // decay sum of each segment (kWT)
  grid_launch_dependents();  // the replay's CTAs may start copying their tiles
  const int BNG = p.B * p.NG;
  const int bg = blockIdx.x >> 2;
  const int ch = threadIdx.x % CH;
  const int cl = (blockIdx.x & 3) * CH + ch;
  const int sg = threadIdx.x / CH;
  const int b = bg / p.NG, c = (bg % p.NG) * CG + cl;
  const float w = (!kWT && c < p.C) ? __ldg(p.w + c) : 0.f;
  const int ntot = p.nch - 1;
  const int per = (ntot + SEG - 1) / SEG;
  const int q0 = min(ntot, sg * per), q1 = min(ntot, q0 + per);
  const float fL = (float)L;
  const float4* tot_of = p.agg_a + (size_t)bg * CG + cl;  // chunk q's total at tot_of[q * BNG * CG]
  const float* wtot_of = kWT ? p.wtot + (size_t)bg * CG + cl : nullptr;
  const size_t qs = (size_t)BNG * CG;
  const size_t n_x0 = (size_t)p.nch * qs;  // x0 entries (bounds-checked build)
  (void)n_x0;
  // one combine of a chunk total (its decay sum wq with per-token decays)
  auto comb = [&](const Acc& x, const float4& t, float wq) {
    return kWT ? combine_wt(x, acc_unpack(t), wq) : combine(x, acc_unpack(t), fL, w);
  };
  grid_wait_prerequisites();  // the totals pass has finished
  // 1. this segment's total; a segment of at most 8 totals stays in registers
  // for step 3
  const bool cached = q1 - q0 <= 8;
  float4 a0[8];
  float w0[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (cached && q0 + r < q1) {
      a0[r] = ldg_f4(tot_of + (q0 + r) * qs);
      w0[r] = kWT ? __ldg(wtot_of + (q0 + r) * qs) : 0.f;
    }
  }
  Acc tot = acc_empty();
  float wseg = 0.f;
  if (cached) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (q0 + r < q1) {
        tot = comb(tot, a0[r], w0[r]);
        wseg += w0[r];
      }
    }
  } else {
    for (int qq = q0; qq < q1; qq += 8) {
      float4 a[8];
      float wa[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (qq + r < q1) {
          a[r] = ldg_f4(tot_of + (qq + r) * qs);
          wa[r] = kWT ? __ldg(wtot_of + (qq + r) * qs) : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (qq + r < q1) {
          tot = comb(tot, a[r], wa[r]);
          wseg += wa[r];
        }
      }
    }
  }
  seg_st[sg][ch] = acc_pack(tot);
  seg_w[sg][ch] = wseg;
  __syncthreads();
  // 2. incoming state of every segment (state in, then the segments before)
  if (sg == 0) {
    Acc x = state_in_acc(p, b, c);
    for (int k = 0; k < SEG; ++k) {
      const Acc t = acc_unpack(seg_st[k][ch]);
      const int kq0 = min(ntot, k * per), kq1 = min(ntot, kq0 + per);
      seg_st[k][ch] = acc_pack(x);
      x = kWT ? combine_wt(x, t, seg_w[k][ch]) : combine(x, t, (float)(kq1 - kq0) * fL, w);
    }
  }
  __syncthreads();
  // 3. incoming state of every chunk of the segment (and of the last chunk)
  Acc x = acc_unpack(seg_st[sg][ch]);
  float4* x0_of = p.x0 + (size_t)bg * CG + cl;
  if (cached) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (q0 + r < q1) {
        if (WKV_IN(p.hdr, (size_t)bg * CG + cl + (q0 + r) * qs, n_x0)) x0_of[(q0 + r) * qs] = acc_pack(x);
        x = comb(x, a0[r], w0[r]);
      }
    }
  } else {
    for (int qq = q0; qq < q1; qq += 8) {
      float4 a[8];
      float wa[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (qq + r < q1) {
          a[r] = ldg_f4(tot_of + (qq + r) * qs);
          wa[r] = kWT ? __ldg(wtot_of + (qq + r) * qs) : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (qq + r < q1) {
          if (WKV_IN(p.hdr, (size_t)bg * CG + cl + (qq + r) * qs, n_x0)) x0_of[(qq + r) * qs] = acc_pack(x);
          x = comb(x, a[r], wa[r]);
        }
      }
    }
  }
  if (((q0 < q1 && q1 == ntot) || (ntot == 0 && sg == 0)) &&
      WKV_IN(p.hdr, (size_t)bg * CG + cl + (size_t)ntot * qs, n_x0))
    x0_of[ntot * qs] = acc_pack(x);
}

// ---------------------------------------------------------------------------
// pipelined single-launch chunked scan (persistent, warp-specialised)
// ---------------------------------------------------------------------------
//
// The same tiles, look-back and arithmetic as wkv_fwd_chunk, but CTAs are
// persistent (one or a few per SM) and take tiles in ticket order, streaming
// them through a ring of p.stages shared-memory stages. Four warp roles, each
// walking the tiles of its CTA in order:
//   producer warp   takes the next ticket and copies the tile's k and v boxes
//                   into the next free stage (TMA, mbarriers);
//   fold warps      (NC, J tokens each) fold the tile into span aggregates as
//                   soon as it has landed; the last of them forms the tile
//                   total and publishes it at once;
//   look-back warp  gathers the tile's incoming state from earlier chunks,
//                   publishes the group prefix where due, and marks the stage
//                   ready for replay;
//   replay warps    (NC, J tokens each) replay the tile from (incoming state +
//                   in-tile prefix), write the outputs and free the stage.
// Folding never waits for a replay, so the totals that every look-back needs
// appear at the speed the data arrives, and the ring's depth bounds how far
// the folds run ahead. Every dependency of a tile is on tiles with smaller
// tickets, so the tile with the smallest unfinished ticket can always proceed.
// Every wait is bounded; a wait that gives up sets the status word and the
// CTA stops taking tiles.
//
// Shared memory: [stages][k | v][L][64] tiles, then float4 agg[stages][NC][64],
// tot[stages][64], xin[stages][64], then four mbarriers per stage, the stage
// tile numbers and an abort flag.
template <int NC>
__host__ __device__ constexpr size_t pipe_aux_bytes(int stages) {
  return sizeof(float4) * 64 * (size_t)stages * (NC + 2) + sizeof(uint64_t) * 4 * stages + sizeof(int) * (stages + 1);
}

__device__ __forceinline__ void pipe_fail(const FwdParams& p, volatile int* abort_flag, int lane) {
  if (lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
  *abort_flag = 1;
}

template <typename KV, typename OUT, int NC, int J>
__global__ void __launch_bounds__((2 * NC + 2) * 32)
    wkv_fwd_pipe(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  constexpr int VEC = 2;
  constexpr int CG = 64;
  constexpr int L = NC * J;
  constexpr int kTile = L * CG;
  constexpr uint32_t kStage = 2u * kTile * (uint32_t)sizeof(KV);
  constexpr int kReplay0 = NC, kLookback = 2 * NC, kProducer = 2 * NC + 1;  // fold warps: 0 .. NC-1
  const int S = p.stages;
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* tiles = reinterpret_cast<KV*>(smem);                            // [S][k|v][L][CG]
  float4* agg = reinterpret_cast<float4*>(smem + (size_t)S * kStage);  // [S][NC][CG]
  float4* tot = agg + (size_t)S * NC * CG;                             // [S][CG]
  float4* xin = tot + (size_t)S * CG;                                  // [S][CG]
  uint64_t* full = reinterpret_cast<uint64_t*>(xin + (size_t)S * CG);  // [S] copy landed
  uint64_t* folded = full + S;                                         // [S] aggregates and total ready
  uint64_t* ready = folded + S;                                        // [S] incoming state ready
  uint64_t* empty = ready + S;                                         // [S] replayed, stage free
  int* tile_id = reinterpret_cast<int*>(empty + S);                    // [S]
  volatile int* abort_flag = tile_id + S;

  const int lane = threadIdx.x & 31;
  const int wp = threadIdx.x >> 5;
  const int T = p.T, C = p.C;
  const int BNG = p.B * p.NG;
  const int cl = lane * VEC;
  const uint32_t target = *reinterpret_cast<volatile uint32_t*>(&p.hdr->epoch) + 1u;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&folded[i], 1);
      mbar_init(&ready[i], 1);
      mbar_init(&empty[i], NC);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (wp == kProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int n = 0;
      for (;; ++n) {
        const int s = n % S;
        if (n >= S && !mbar_wait(&empty[s], ((n / S) - 1) & 1, p.timeout_ns)) pipe_fail(p, abort_flag, 0);
        const int t = *abort_flag ? p.n_tiles : (int)atomicAdd(&p.hdr->ticket, 1u);
        if (t >= p.n_tiles) {
          // the previous copy into this stage must have landed before the
          // stage's next phase marks the end of the stream
          if (n >= S && !mbar_wait(&full[s], ((n / S) - 1) & 1, p.timeout_ns))
            atomicOr(&p.hdr->status, kStatusWaitTimeout);
          tile_id[s] = t;
          mbar_arrive(&full[s]);  // end of the stream for the other warps
          break;
        }
        tile_id[s] = t;
        const int j = t / BNG, bg = t % BNG;
        mbar_arrive_expect_tx(&full[s], kStage);
        tma_load_3d(tiles + (size_t)s * 2 * kTile, &tmk, &full[s], (bg % p.NG) * CG, j * L, bg / p.NG);
        tma_load_3d(tiles + (size_t)s * 2 * kTile + kTile, &tmv, &full[s], (bg % p.NG) * CG, j * L, bg / p.NG);
      }
      // no copy may still be writing into shared memory when the CTA exits
      // (the stage of the end marker was drained above)
      for (int m = max(0, n - S + 1); m < n; ++m)
        if (!mbar_wait(&full[m % S], (m / S) & 1, p.timeout_ns)) atomicOr(&p.hdr->status, kStatusWaitTimeout);
    }
  } else if (wp == kLookback) {
    // ----------------------------------------------------------- look-back
    for (int n = 0;; ++n) {
      const int s = n % S;
      const uint32_t ph = (n / S) & 1;
      if (!mbar_wait(&full[s], ph, p.timeout_ns)) {
        pipe_fail(p, abort_flag, lane);
        break;
      }
      const int tile = tile_id[s];
      if (tile >= p.n_tiles) {  // end of the stream: pass it on to the replay warps
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[s]);
        break;
      }
      const int j = tile / BNG, bg = tile % BNG;
      const int b = bg / p.NG, c0 = (bg % p.NG) * CG + cl;
      float w[VEC];
      Acc x[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) w[e] = (c0 + e < C) ? __ldg(p.w + c0 + e) : 0.f;
      // The incoming state needs nothing from this tile. Only chunk 0 reads
      // the state in; its published total already contains it, so no later
      // tile reads the caller's state (which state_out may alias).
      const int qb = j / p.G;
      const int first = qb * p.G;
#pragma unroll
      for (int e = 0; e < VEC; ++e) x[e] = (j == 0) ? state_in_acc(p, b, c0 + e) : acc_empty();
      if (j > 0) {
        const uint32_t* fp = p.flags_p + (size_t)(qb - 1) * BNG + bg;
        bool got = false;
        uint64_t tstart = 0;
        while (true) {
          bool all = (qb == 0) || ld_relaxed_u32(fp) == target;
          for (int jj = first + lane; jj < j; jj += 32)
            all &= ld_relaxed_u32(p.flags_a + (size_t)jj * BNG + bg) == target;
          all = __all_sync(0xffffffffu, all);
          if (all) {
            got = true;
            break;
          }
          if (tstart == 0) {
            tstart = global_ns();
          } else if (global_ns() - tstart > p.timeout_ns) {
            break;
          }
          __nanosleep(32);
        }
        if (!got && lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
        fence_acq_rel_gpu();
        gather_group<VEC, CG, L>(p, x, first, j, bg, cl, w, qb > 0, qb);
      }
      // the replay also needs this tile's aggregates: wait for its fold
      if (!mbar_wait(&folded[s], ph, p.timeout_ns)) {
        pipe_fail(p, abort_flag, lane);
        break;
      }
      if (j != p.nch - 1 && (j % p.G) == p.G - 1) {
        // the last chunk of a look-back group publishes its inclusive prefix
        float4* dst = p.agg_p + ((size_t)qb * BNG + bg) * CG + cl;
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          dst[e] = acc_pack(combine(x[e], acc_unpack(tot[(size_t)s * CG + cl + e]), (float)L, w[e]));
        __threadfence();
        __syncwarp();
        if (lane == 0 && tile != p.inject_tile) st_release_u32(p.flags_p + (size_t)qb * BNG + bg, target);
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) xin[(size_t)s * CG + cl + e] = acc_pack(x[e]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);
    }
  } else if (wp < kReplay0) {
    // --------------------------------------------------------------- fold
    for (int n = 0;; ++n) {
      const int s = n % S;
      const bool got = mbar_wait(&full[s], (n / S) & 1, p.timeout_ns);
      const int tile = got ? tile_id[s] : p.n_tiles;
      if (named_sync_or<NC * 32>(1, !got || *abort_flag != 0)) {
        pipe_fail(p, abort_flag, lane);
        break;
      }
      if (tile >= p.n_tiles) break;
      const int j = tile / BNG, bg = tile % BNG;
      const int c0 = (bg % p.NG) * CG + cl;
      const int nv = max(0, min(J, T - (j * L + wp * J)));
      float w[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) w[e] = (c0 + e < C) ? __ldg(p.w + c0 + e) : 0.f;
      const KV* ks = tiles + (size_t)s * 2 * kTile + (wp * J) * CG + cl;
      Acc a[VEC];
      aggregate_tile_span<KV, J, VEC, CG>(ks, ks + kTile, nv, w, a);
      float4* ag = agg + (size_t)s * NC * CG;
#pragma unroll
      for (int e = 0; e < VEC; ++e) ag[wp * CG + cl + e] = acc_pack(a[e]);
      named_sync<NC * 32>(1);
      if (wp == NC - 1) {
        // the tile total: published at once, and kept for the group prefix
        Acc tt[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) tt[e] = acc_empty();
        for (int qq = 0; qq < NC - 1; ++qq) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) tt[e] = combine(tt[e], acc_unpack(ag[qq * CG + cl + e]), (float)J, w[e]);
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          tt[e] = combine(tt[e], a[e], (float)nv, w[e]);
          tot[(size_t)s * CG + cl + e] = acc_pack(tt[e]);
        }
        if (j != p.nch - 1 && WKV_IN(p.hdr, (size_t)tile * CG + cl + VEC - 1, (size_t)p.n_tiles * CG)) {
          const int b = bg / p.NG;
          float4* dst = p.agg_a + (size_t)tile * CG + cl;
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            dst[e] = acc_pack(j == 0 ? combine(state_in_acc(p, b, c0 + e), tt[e], (float)L, w[e]) : tt[e]);
          __threadfence();
          __syncwarp();
          if (lane == 0 && tile != p.inject_tile) st_release_u32(p.flags_a + tile, target);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&folded[s]);
      }
    }
  } else {
    // ------------------------------------------------------------- replay
    const int r = wp - kReplay0;  // this warp's span of every tile
    for (int n = 0;; ++n) {
      const int s = n % S;
      if (!mbar_wait(&ready[s], (n / S) & 1, p.timeout_ns)) {
        pipe_fail(p, abort_flag, lane);
        break;
      }
      const int tile = tile_id[s];
      if (tile >= p.n_tiles || *abort_flag) break;
      const int j = tile / BNG, bg = tile % BNG;
      const int b = bg / p.NG, c0 = (bg % p.NG) * CG + cl;
      const int ts = j * L + r * J;
      const int nv = max(0, min(J, T - ts));
      const bool last_chunk = (j == p.nch - 1);
      const int p_last = last_chunk ? (T - 1 - j * L) / J : NC - 1;
      if (nv > 0 && WKV_IN(p.hdr, (size_t)b * T + ts + nv - 1, (size_t)p.B * T)) {
        float w[VEC], u[VEC], cb[VEC];
        bool fast = true;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const bool okc = c0 + e < C;
          w[e] = okc ? __ldg(p.w + c0 + e) : 0.f;
          u[e] = okc ? __ldg(p.u + c0 + e) : 0.f;
          fast &= fast_uw(u[e], w[e]);
          cb[e] = ex2(fminf(fmaxf(u[e] - w[e], -kFastUW), kFastUW) * kLog2e);
        }
        fast = __all_sync(0xffffffffu, fast);
        // state at the start of the span: incoming state, then the spans before it
        const float4* ag = agg + (size_t)s * NC * CG;
        Acc st[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) st[e] = acc_empty();
        for (int qq = 0; qq < r; ++qq) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) st[e] = combine(st[e], acc_unpack(ag[qq * CG + cl + e]), (float)J, w[e]);
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          st[e] = combine(acc_unpack(xin[(size_t)s * CG + cl + e]), st[e], (float)(r * J), w[e]);
        const KV* ks = tiles + (size_t)s * 2 * kTile + (r * J) * CG + cl;
        const KV* vs = ks + kTile;
        OUT* orow = reinterpret_cast<OUT*>(p.out) + ((size_t)b * T + ts) * C + c0;
        const bool lane_vec = p.vec_store != 0 && c0 + VEC <= C;
        if (fast && nv == J) {
          constexpr int NB = J < 8 ? J : 8;  // tokens per block of step_tokens
#pragma unroll
          for (int i0 = 0; i0 < J; i0 += NB) {
            float kb[NB][VEC], vb[NB][VEC], ob[NB][VEC];
#pragma unroll
            for (int ii = 0; ii < NB; ++ii) {
              load_vec<KV, VEC>(ks + (i0 + ii) * CG, kb[ii]);
              load_vec<KV, VEC>(vs + (i0 + ii) * CG, vb[ii]);
            }
            step_tokens<NB, VEC>(st, kb, vb, w, cb, ob);
#pragma unroll
            for (int ii = 0; ii < NB; ++ii) {
              gate_row<KV, VEC>(p, ((size_t)b * T + ts + i0 + ii) * C, c0, ob[ii]);
              if (lane_vec) {
                stg_stream<OUT, VEC>(orow + (size_t)(i0 + ii) * C, ob[ii]);
              } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                  if (c0 + e < C) orow[(size_t)(i0 + ii) * C + e] = Elem<OUT>::from_f32(ob[ii][e]);
              }
            }
          }
        } else {
          for (int i = 0; i < nv; ++i) {
            float kx[VEC], vx[VEC], o[VEC];
            load_vec<KV, VEC>(ks + i * CG, kx);
            load_vec<KV, VEC>(vs + i * CG, vx);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              if (fast) {
                o[e] = step_token(st[e], kx[e], vx[e], w[e], cb[e]);
              } else {
                o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
                add_token(st[e], kx[e], vx[e], w[e]);
              }
            }
            gate_row<KV, VEC>(p, ((size_t)b * T + ts + i) * C, c0, o);
#pragma unroll
            for (int e = 0; e < VEC; ++e)
              if (c0 + e < C) orow[(size_t)i * C + e] = Elem<OUT>::from_f32(o[e]);
          }
        }
        if (last_chunk && r == p_last && p.o_num) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            if (c0 + e < C) {
              const size_t i = (size_t)b * C + c0 + e;
              p.o_num[i] = st[e].num;
              p.o_den[i] = st[e].den;
              p.o_max[i] = acc_max_e(st[e], w[e]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the stage may be refilled
    }
  }

  // ---- hand the workspace back for the next launch once every CTA is done
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&p.hdr->done, 1u);
    if (prev == gridDim.x - 1) {
      p.hdr->ticket = 0;
      p.hdr->done = 0;
      __threadfence();
      atomicExch(&p.hdr->epoch, target);
    }
  }
}

}  // namespace wkv
