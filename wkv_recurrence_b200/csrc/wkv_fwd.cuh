// Forward kernels of the WKV operator over [B, T, C] sequences.
//
// Both kernels stream k and v through shared memory with TMA (3-D tiled bulk
// copies of a [tokens x channel-group] box, completion on an mbarrier) and run
// the recurrence of "Linear attention without writing a CUDA kernel", section
// "The recurrence", in the anchored form of wkv_device.cuh, one channel per
// register lane, VEC adjacent channels per thread.
//
// * wkv_fwd_seq: one CTA per (batch row, channel group), walking all T tokens
//   through a STAGES-deep ring of [LT x CG] tiles. For many channels (B*C
//   large): the state never leaves registers.
//
// * wkv_fwd_chunk: for few channels and long T. T is cut into chunks of
//   L = P*J tokens; a tile is (chunk, batch row, channel group). Persistent
//   CTAs take tiles in order from a ticket counter, so every tile a CTA waits
//   for was handed out earlier to a running CTA. Per tile:
//     1. P sub-chunks of J tokens each (one warp-row of threads per sub-chunk)
//        fold their tokens from the empty state into an aggregate;
//     2. one row of threads combines the P aggregates into the tile total,
//        publishes it, and forms the tile's incoming state from the chunks
//        before it (look-back, below);
//     3. every sub-chunk replays its tokens from its incoming state, still in
//        shared memory, and writes the outputs.
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
  float4* agg_p;       // [nblk * B * NG][CG]
};

template <typename OUT, int VEC>
__device__ __forceinline__ void store_out(OUT* row, int c0, int C, bool vec_ok, const float (&o)[VEC]) {
  if (vec_ok && c0 + VEC <= C) {
    store_vec<OUT, VEC>(row + c0, o);
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e)
      if (c0 + e < C) row[c0 + e] = Elem<OUT>::from_f32(o[e]);
  }
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
template <typename KV, typename OUT, int VEC, int THREADS, int LT, int STAGES, bool kTMA>
__global__ void __launch_bounds__(THREADS)
    wkv_fwd_seq(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  constexpr int CG = THREADS * VEC;
  constexpr int kTile = LT * CG;  // elements per tensor per stage
  constexpr uint32_t kStageBytes = 2u * kTile * sizeof(KV);
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* tiles = reinterpret_cast<KV*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);

  const int tid = threadIdx.x;
  const int b = blockIdx.x / p.NG;
  const int g = blockIdx.x % p.NG;
  const int T = p.T, C = p.C;
  const int c0 = g * CG + tid * VEC;
  const int ntile = (T + LT - 1) / LT;

  if (kTMA && tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    for (int s = 0; s < STAGES && s < ntile; ++s) {
      mbar_arrive_expect_tx(&full[s], kStageBytes);
      tma_load_3d(tiles + (2 * s) * kTile, &tmk, &full[s], g * CG, s * LT, b);
      tma_load_3d(tiles + (2 * s + 1) * kTile, &tmv, &full[s], g * CG, s * LT, b);
    }
  }

  float w[VEC], u[VEC];
  Acc st[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const int c = c0 + e;
    const bool ok = c < C;
    w[e] = ok ? p.w[c] : 0.f;
    u[e] = ok ? p.u[c] : 0.f;
    st[e] = acc_empty();
    if (ok && p.s_num) {
      const size_t i = (size_t)b * C + c;
      st[e] = acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
    }
  }
  __syncthreads();

  OUT* out = reinterpret_cast<OUT*>(p.out);
  const bool vec_ok = p.vec_store != 0;
  int issued = (STAGES < ntile) ? STAGES : ntile;  // tiles whose loads were issued
  int aborted_at = -1;
  for (int i = 0; i < ntile; ++i) {
    const int s = kTMA ? (i % STAGES) : 0;
    const int t0 = i * LT;
    if (kTMA) {
      const bool ok = mbar_wait(&full[s], (i / STAGES) & 1, p.timeout_ns);
      if (__syncthreads_or(!ok)) {
        aborted_at = i;
        break;
      }
    } else {
      coop_load_tile<KV>(tiles, reinterpret_cast<const KV*>(p.k), b, t0, LT, g * CG, CG, T, C);
      coop_load_tile<KV>(tiles + kTile, reinterpret_cast<const KV*>(p.v), b, t0, LT, g * CG, CG, T, C);
      __syncthreads();
    }
    const KV* ks = tiles + (2 * s) * kTile + tid * VEC;
    const KV* vs = ks + kTile;
    const int nv = min(LT, T - t0);
    OUT* orow = out + ((size_t)b * T + t0) * C;
    if (c0 < C) {
      if (nv == LT) {
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
          store_out<OUT, VEC>(orow + (size_t)j * C, c0, C, vec_ok, o);
        }
      }
    }
    __syncthreads();  // every thread is done with stage s
    if (kTMA && tid == 0 && i + STAGES < ntile) {
      fence_proxy_async_smem();
      const int tn = (i + STAGES) * LT;
      mbar_arrive_expect_tx(&full[s], kStageBytes);
      tma_load_3d(tiles + (2 * s) * kTile, &tmk, &full[s], g * CG, tn, b);
      tma_load_3d(tiles + (2 * s + 1) * kTile, &tmv, &full[s], g * CG, tn, b);
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

  if (p.o_num && c0 < C) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const int c = c0 + e;
      if (c < C) {
        const size_t i = (size_t)b * C + c;
        p.o_num[i] = st[e].num;
        p.o_den[i] = st[e].den;
        p.o_max[i] = acc_max_e(st[e], w[e]);
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
__device__ __forceinline__ void row_sync() {
  // barrier among the first N threads of the CTA (whole warps)
  if (N == 32) {
    __syncwarp();
  } else {
    asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
  }
}

template <typename KV, typename OUT, int VEC, int RW, int P, int J, bool kTMA>
__global__ void __launch_bounds__(RW * P)
    wkv_fwd_chunk(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  static_assert(RW % 32 == 0, "a row of threads is whole warps");
  constexpr int CG = RW * VEC;  // channels per tile
  constexpr int L = P * J;      // tokens per tile
  constexpr int kTile = L * CG;
  constexpr uint32_t kStageBytes = 2u * kTile * sizeof(KV);
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* tiles = reinterpret_cast<KV*>(smem);                                 // [2 stages][k,v][L][CG]
  float4* buf = reinterpret_cast<float4*>(smem + 2 * kStageBytes);          // [P][CG]
  uint64_t* full = reinterpret_cast<uint64_t*>(buf + P * CG);               // [2]
  int* tile_id = reinterpret_cast<int*>(full + 2);                          // [2]

  const int tid = threadIdx.x;
  const int pr = tid / RW;  // sub-chunk of this thread
  const int rr = tid % RW;  // position in the row
  const int T = p.T, C = p.C;
  const int BNG = p.B * p.NG;
  const uint32_t target = *reinterpret_cast<volatile uint32_t*>(&p.hdr->epoch) + 1u;
  OUT* out = reinterpret_cast<OUT*>(p.out);
  const bool vec_ok = p.vec_store != 0;

  if (tid == 0) {
    if (kTMA) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
      mbar_init(&full[0], 1);
      mbar_init(&full[1], 1);
      fence_mbar_init();
    }
    const int t = (int)atomicAdd(&p.hdr->ticket, 1u);
    tile_id[0] = t;
    if (kTMA && t < p.n_tiles) {
      const int j = t / BNG, bg = t % BNG;
      mbar_arrive_expect_tx(&full[0], kStageBytes);
      tma_load_3d(tiles, &tmk, &full[0], (bg % p.NG) * CG, j * L, bg / p.NG);
      tma_load_3d(tiles + kTile, &tmv, &full[0], (bg % p.NG) * CG, j * L, bg / p.NG);
    }
  }
  __syncthreads();

  bool timed_out = false;
  int stuck_it = -1;  // iteration whose copy did not arrive in time, if any
  for (int it = 0;; ++it) {
    const int slot = it & 1;             // ticket slot (and stage, with TMA)
    const int s = kTMA ? slot : 0;       // shared-memory stage
    const int tile = tile_id[slot];
    if (tile >= p.n_tiles) break;
    const int j = tile / BNG;
    const int bg = tile % BNG;
    const int b = bg / p.NG, g = bg % p.NG;
    const int t0 = j * L;
    const int cbase = g * CG;

    if (tid == 0) {  // hand out and prefetch the next tile
      const int tn = (int)atomicAdd(&p.hdr->ticket, 1u);
      tile_id[slot ^ 1] = tn;
      if (kTMA && tn < p.n_tiles) {
        const int jn = tn / BNG, bgn = tn % BNG;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[s ^ 1], kStageBytes);
        tma_load_3d(tiles + (2 * (s ^ 1)) * kTile, &tmk, &full[s ^ 1], (bgn % p.NG) * CG, jn * L, bgn / p.NG);
        tma_load_3d(tiles + (2 * (s ^ 1) + 1) * kTile, &tmv, &full[s ^ 1], (bgn % p.NG) * CG, jn * L,
                    bgn / p.NG);
      }
    }

    if (kTMA) {
      const bool ok = mbar_wait(&full[s], (it >> 1) & 1, p.timeout_ns);
      if (__syncthreads_or(!ok)) {
        timed_out = true;
        stuck_it = it;
        break;
      }
    } else {
      coop_load_tile<KV>(tiles, reinterpret_cast<const KV*>(p.k), b, t0, L, cbase, CG, T, C);
      coop_load_tile<KV>(tiles + kTile, reinterpret_cast<const KV*>(p.v), b, t0, L, cbase, CG, T, C);
      __syncthreads();
    }

    const KV* ks = tiles + (2 * s) * kTile + rr * VEC;
    const KV* vs = ks + kTile;
    const int cl = rr * VEC;       // channel offset inside the group
    const int c0 = cbase + cl;     // first channel of this thread
    float w[VEC], u[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const bool ok = c0 + e < C;
      w[e] = ok ? __ldg(p.w + c0 + e) : 0.f;
      u[e] = ok ? __ldg(p.u + c0 + e) : 0.f;
    }
    const bool last_chunk = (j == p.nch - 1);
    const int ts = t0 + pr * J;                       // first token of this sub-chunk
    const int nv = max(0, min(J, T - ts));            // its tokens
    const int p_last = last_chunk ? (T - 1 - t0) / J : P - 1;

    // 1. sub-chunk aggregates from the empty state
    {
      Acc a[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) a[e] = acc_empty();
      if (!(last_chunk && pr >= p_last)) {
        if (nv == J) {
#pragma unroll 4
          for (int jj = 0; jj < J; ++jj) {
            float kx[VEC], vx[VEC];
            load_vec<KV, VEC>(ks + (pr * J + jj) * CG, kx);
            load_vec<KV, VEC>(vs + (pr * J + jj) * CG, vx);
#pragma unroll
            for (int e = 0; e < VEC; ++e) add_token(a[e], kx[e], vx[e], w[e]);
          }
        } else {
          for (int jj = 0; jj < nv; ++jj) {
            float kx[VEC], vx[VEC];
            load_vec<KV, VEC>(ks + (pr * J + jj) * CG, kx);
            load_vec<KV, VEC>(vs + (pr * J + jj) * CG, vx);
#pragma unroll
            for (int e = 0; e < VEC; ++e) add_token(a[e], kx[e], vx[e], w[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) buf[pr * CG + cl + e] = acc_pack(a[e]);
    }
    __syncthreads();

    // 2. tile total, publication, look-back, sub-chunk prefixes (row 0 only)
    if (pr == 0) {
      Acc tot[VEC], x[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) tot[e] = acc_unpack(buf[cl + e]);
      for (int q = 1; q < P; ++q) {
        const float len = (float)max(0, min(J, T - (t0 + q * J)));
#pragma unroll
        for (int e = 0; e < VEC; ++e) tot[e] = combine(tot[e], acc_unpack(buf[q * CG + cl + e]), len, w[e]);
      }
      const bool inject = (tile == p.inject_tile);
      if (!last_chunk) {
        float4* dst = p.agg_a + (size_t)tile * CG + cl;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc_pack(tot[e]);
        __threadfence();
        row_sync<RW>();
        if (rr == 0 && !inject) st_release_u32(p.flags_a + tile, target);
      }

      // incoming state of the tile
      const int qb = j / p.G;
      const int first = qb * p.G;  // first chunk of this look-back group
      if (qb == 0) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          x[e] = acc_empty();
          if (p.s_num && c0 + e < C) {
            const size_t i = (size_t)b * C + c0 + e;
            x[e] = acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
          }
        }
      }
      if (j > 0) {
        // wait until every flag this tile needs is set
        const uint32_t* fp = p.flags_p + (size_t)(qb - 1) * BNG + bg;
        bool ready = false;
        uint64_t tstart = 0;
        while (true) {
          bool all = (qb == 0) || ld_relaxed_u32(fp) == target;
          for (int jj = first; jj < j; ++jj) all &= ld_relaxed_u32(p.flags_a + (size_t)jj * BNG + bg) == target;
          if (all) {
            ready = true;
            break;
          }
          if (tstart == 0) {
            tstart = global_ns();
          } else if (global_ns() - tstart > p.timeout_ns) {
            break;
          }
          __nanosleep(64);
        }
        if (!ready) timed_out = true;
        fence_acq_rel_gpu();
        if (qb > 0) {
          const float4* src = p.agg_p + ((size_t)(qb - 1) * BNG + bg) * CG + cl;
#pragma unroll
          for (int e = 0; e < VEC; ++e) x[e] = acc_unpack(ld_relaxed_f4(src + e));
        }
        for (int jj = first; jj < j; ++jj) {
          const float4* src = p.agg_a + ((size_t)jj * BNG + bg) * CG + cl;
#pragma unroll
          for (int e = 0; e < VEC; ++e) x[e] = combine(x[e], acc_unpack(ld_relaxed_f4(src + e)), (float)L, w[e]);
        }
      }
      // the last chunk of a group publishes its inclusive prefix
      if (!last_chunk && (j % p.G) == p.G - 1) {
        float4* dst = p.agg_p + ((size_t)qb * BNG + bg) * CG + cl;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc_pack(combine(x[e], tot[e], (float)L, w[e]));
        __threadfence();
        row_sync<RW>();
        if (rr == 0 && !inject) st_release_u32(p.flags_p + (size_t)qb * BNG + bg, target);
      }
      // incoming state of every sub-chunk
      for (int q = 0; q < P; ++q) {
        const float len = (float)max(0, min(J, T - (t0 + q * J)));
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const Acc a = acc_unpack(buf[q * CG + cl + e]);
          buf[q * CG + cl + e] = acc_pack(x[e]);
          x[e] = combine(x[e], a, len, w[e]);
        }
      }
    }
    __syncthreads();

    // 3. replay each sub-chunk from its incoming state and write the outputs
    {
      Acc st[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) st[e] = acc_unpack(buf[pr * CG + cl + e]);
      OUT* orow = out + ((size_t)b * T + ts) * C;
      if (c0 < C) {
        if (nv == J) {
#pragma unroll 4
          for (int jj = 0; jj < J; ++jj) {
            float kx[VEC], vx[VEC], o[VEC];
            load_vec<KV, VEC>(ks + (pr * J + jj) * CG, kx);
            load_vec<KV, VEC>(vs + (pr * J + jj) * CG, vx);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
              add_token(st[e], kx[e], vx[e], w[e]);
            }
            store_out<OUT, VEC>(orow + (size_t)jj * C, c0, C, vec_ok, o);
          }
        } else {
          for (int jj = 0; jj < nv; ++jj) {
            float kx[VEC], vx[VEC], o[VEC];
            load_vec<KV, VEC>(ks + (pr * J + jj) * CG, kx);
            load_vec<KV, VEC>(vs + (pr * J + jj) * CG, vx);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              o[e] = out_token(st[e], kx[e], vx[e], w[e], u[e]);
              add_token(st[e], kx[e], vx[e], w[e]);
            }
            store_out<OUT, VEC>(orow + (size_t)jj * C, c0, C, vec_ok, o);
          }
        }
        if (last_chunk && pr == p_last && p.o_num) {
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
    }
    __syncthreads();  // stage s and buf are free again
  }

  // leave: report, drain a copy still in flight (bounded), hand the workspace
  // back for the next launch
  if (timed_out) atomicOr(&p.hdr->status, kStatusWaitTimeout);
  if (kTMA && tid == 0 && stuck_it >= 0) {
    // the late copy, and the prefetch issued in the same iteration: bounded
    (void)mbar_wait(&full[stuck_it & 1], (stuck_it >> 1) & 1, p.timeout_ns);
    const int nx = stuck_it + 1;
    if (tile_id[nx & 1] < p.n_tiles) (void)mbar_wait(&full[nx & 1], (nx >> 1) & 1, p.timeout_ns);
  }
  __syncthreads();
  if (tid == 0) {
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
