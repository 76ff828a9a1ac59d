// The chunked scan over T in thread-block clusters, reading k and v from HBM
// once.
//
// A cluster of ncl CTAs (at most kClusterMaxCTAs) takes one SEGMENT of ncl * NW * J tokens
// of one (batch row, 32-channel group); CTA `rank` holds tokens
// [rank*TPC, (rank+1)*TPC) of the segment (TPC = NW*J), one span of J tokens
// per warp, one channel per lane. Each warp streams its span through a ring of
// its own: NS shared-memory stages of LB tokens x 32 channels of k and v (and
// w_t), copied by TMA and completing on one mbarrier per stage. The span goes
// through the ring twice:
//   1. fold: block by block from HBM, each block folded in registers (largest
//      end-of-block exponent first, then the weighted sums) and combined into
//      the span's aggregate;
//   2. prefixes: each warp combines the aggregates of the warps before it
//      (shared memory), the last warp forms the CTA's total, and after a
//      cluster barrier each CTA combines the totals of the CTAs before it
//      (distributed shared memory); the segment's incoming state is the state
//      in for the first segment, else the inclusive prefix that the previous
//      segment of the same channel group published in global memory (flag +
//      payload, a bounded wait); the last CTA publishes this segment's
//      inclusive prefix at once;
//   3. replay: the same blocks again, from L2, where the fold left them
//      moments before (the ring's first replay copies are in flight during
//      step 2), gated by sigmoid(r) when r is given; the warp holding token
//      T-1 writes the state out.
// Segments take their work item from a ticket counter in segment-major order,
// so a segment's predecessor (same channel group, previous segment) always
// took its ticket earlier: every wait is for a cluster that is running or
// done. With a single segment there is no ticket and no wait.
//
// The order of every combine depends on the shape only (bitwise
// reproducible). With kWT the decay is per token ("RWKV-v6 Architecture",
// section "2. Dynamic Data-Dependent Decay"): w_t comes through the ring with
// k and v and the combines carry each block's and span's decay sum.
//
// The state in is read by the first segment's CTAs, and the state out is
// written by the last segment, which (through the published prefixes, or the
// cluster barrier when there is one segment) runs after those reads, so the
// two may alias. A second cluster barrier (arrive after the last remote read,
// wait before exit) keeps every CTA's shared memory alive while others may
// read it. Only the threads whose accesses must be ordered before another
// CTA's (the writes of the ticket and of a CTA's total, the first segment's
// read of the state in) arrive with release semantics, the rest relaxed. All
// threads of every CTA take every barrier; no thread returns
// early, and a warp whose copy wait runs out stops consuming, reports
// kStatusWaitTimeout, and before the end waits (bounded) for the copies it
// still has in flight.
#pragma once

#include "wkv_device.cuh"
#include "wkv_fwd.cuh"

namespace wkv {

// Ring and cluster shape, measured on the long workload (1 x 65536 x 2048
// fp32, 8-warp CTAs, 64-token spans). Clusters of up to 8 CTAs: rings of 4
// stages of 8 tokens 488 us, 2 stages of 16 tokens 418 us (the same shared
// memory in half as many copies), 4 stages of 16 tokens 725 us (twice the
// shared memory, half the CTAs per SM). With 2 stages of 16 tokens, clusters
// of up to 8, 4, 2 and 1 CTAs: 418, 392, 364 and 461 us (1: twice the
// segments per channel group); up to 2 CTAs with 1 stage of 32 tokens: 372 us.
constexpr int kClusterLB = 16;     // tokens per ring stage
constexpr int kClusterNS = 2;      // ring stages per warp
constexpr int kClusterMaxCTAs = 2; // CTAs per cluster (and segment), at most

template <typename KV, bool kWT>
__host__ __device__ constexpr uint32_t cluster_stage_bytes() {
  return (uint32_t)(kClusterLB * 32 * (2 * sizeof(KV) + (kWT ? sizeof(float) : 0)));
}

// Shared-memory bytes of wkv_fwd_cluster.
template <typename KV, int NW, bool kWT>
__host__ __device__ constexpr size_t cluster_smem_bytes() {
  return (size_t)NW * kClusterNS * cluster_stage_bytes<KV, kWT>()  // the warps' rings
         + (size_t)NW * kClusterNS * 8                             // their mbarriers
         + (size_t)NW * 32 * (16 + (kWT ? 4 : 0))                  // span aggregates (and decay sums)
         + 32 * (16 + 4)                                           // the CTA's total and decay sum
         + 32 * (16 + 4)                                           // the segment's incoming state
         + 32 * 16                                                 // the totals of the CTAs before
         + 16;                                                     // the cluster's ticket
}

// Aggregate of n <= J tokens held in registers, anchored at the last one
// (the register twin of aggregate_tile_span): s_i = k_i - (n-1-i) w.
template <int J>
__device__ __forceinline__ Acc fold_regs(const float (&kx)[J], const float (&vx)[J], int n, float w) {
  float M = kNegBig;
  const float last = (float)(n - 1);
#pragma unroll
  for (int i = 0; i < J; ++i)
    if (i < n) M = fmaxf(M, fmaf((float)i - last, w, kx[i]));
  const float ML = M * kLog2e;
  float num = 0.f, den = 0.f;
#pragma unroll
  for (int i = 0; i < J; ++i) {
    if (i < n) {
      const float x = ex2(fmaf(fmaf((float)i - last, w, kx[i]), kLog2e, -ML));
      num = fmaf(x, vx[i], num);
      den += x;
    }
  }
  if (n <= 0) return acc_empty();
  const float corr = fmaf(M, kLog2e, -ML);
  const float fix = fmaf(-corr, 0.6931471805599453f, 1.f);
  return Acc{num * fix, den * fix, M, 0.f};
}

// The same with per-token decays (the register twin of aggregate_span_wt):
// s_i = k_i - (w_{i+1} + ... + w_{n-1}), compensated suffix sums; also the
// span's decay sum.
template <int J>
__device__ __forceinline__ Acc fold_regs_wt(const float (&kx)[J], const float (&vx)[J], const float (&wx)[J], int n,
                                            float& wsum) {
  float sx[J];
  float hi = 0.f, lo = 0.f, M = kNegBig;
#pragma unroll
  for (int i = J - 1; i >= 0; --i) {
    if (i < n) {
      sx[i] = (kx[i] - hi) - lo;
      M = fmaxf(M, sx[i]);
      float h, e;
      two_sum(hi, wx[i], h, e);
      hi = h;
      lo += e;
    }
  }
  wsum = hi + lo;
  const float ML = M * kLog2e;
  float num = 0.f, den = 0.f;
#pragma unroll
  for (int i = 0; i < J; ++i) {
    if (i < n) {
      const float x = ex2(fmaf(sx[i], kLog2e, -ML));
      num = fmaf(x, vx[i], num);
      den += x;
    }
  }
  if (n <= 0) return acc_empty();
  const float corr = fmaf(M, kLog2e, -ML);
  const float fix = fmaf(-corr, 0.6931471805599453f, 1.f);
  return Acc{num * fix, den * fix, M, 0.f};
}

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* q) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(q) : "memory");
  return v;
}

template <typename KV, typename OUT, int NW, int J, bool kWT>
__global__ void __launch_bounds__(NW * 32, (NW == 8 ? 3 : 6))
    wkv_fwd_cluster(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmw) {
  constexpr int CG = 32;
  constexpr int LB = kClusterLB;
  constexpr int NS = kClusterNS;
  constexpr int TPC = NW * J;
  static_assert(J % LB == 0, "a span is whole ring blocks");
  constexpr uint32_t kStage = cluster_stage_bytes<KV, kWT>();
  constexpr int kTile = LB * CG;  // elements per tensor per stage
  extern __shared__ __align__(1024) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int wp = threadIdx.x >> 5;
  unsigned char* ring = smem + (size_t)wp * NS * kStage;                              // this warp's stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NW * NS * kStage) + wp * NS;
  float4* sagg = reinterpret_cast<float4*>(smem + (size_t)NW * NS * (kStage + 8));   // [NW][CG]
  float* swsum = reinterpret_cast<float*>(sagg + NW * CG);                            // [NW][CG] (kWT)
  float4* stot = reinterpret_cast<float4*>(swsum + (kWT ? NW * CG : 0));              // [CG]
  float* stotw = reinterpret_cast<float*>(stot + CG);                                 // [CG]
  float4* sx = reinterpret_cast<float4*>(stotw + CG);                                 // [CG] incoming state
  float* sxw = reinterpret_cast<float*>(sx + CG);                                     // [CG] their decay sum (kWT)
  float4* sxl = reinterpret_cast<float4*>(sxw + CG);                                  // [CG] CTAs before this one
  uint32_t* sticket = reinterpret_cast<uint32_t*>(sxl + CG);

  const int T = p.T, C = p.C;
  const int ncl = p.cluster;
  const int nseg = p.nseg;
  const int rank = (int)(blockIdx.x % (unsigned)ncl);
  const int ngc = (C + CG - 1) / CG;
  const int items = p.B * ngc;
  const uint32_t target = nseg > 1 ? *reinterpret_cast<volatile uint32_t*>(&p.hdr->epoch) + 1u : 0u;

  // ---- the cluster's work item (segment-major ticket order with segments)
  int cl_id;
  if (nseg > 1) {
    if (rank == 0 && threadIdx.x == 0) *sticket = atomicAdd(&p.hdr->ticket, 1u);
    if (rank == 0 && wp == 0) {
      cluster_arrive();  // (release: the ticket)
    } else {
      cluster_arrive_relaxed();
    }
    cluster_wait();
    cl_id = (int)ld_dsmem_u32(map_shared_rank(sticket, 0));
    if (rank == 0 && threadIdx.x == 0) {
      // every cluster has read the epoch and taken its ticket before it counts
      // itself; the last one hands the header back for the next launch
      const uint32_t prev = atomicAdd(&p.hdr->done, 1u);
      if (prev == (uint32_t)(nseg * items) - 1u) {
        p.hdr->ticket = 0;
        p.hdr->done = 0;
        __threadfence();
        atomicExch(&p.hdr->epoch, target);
      }
    }
  } else {
    cl_id = (int)(blockIdx.x / (unsigned)ncl);
  }
  const int seg = cl_id / items, it = cl_id % items;
  const int b = it / ngc, g = it % ngc;
  const int c = g * CG + lane;
  const bool cok = c < C;
  const int t_seg = seg * ncl * TPC;
  const int t_cta = t_seg + rank * TPC;
  const int ts = t_cta + wp * J;                // this warp's span
  const int nv = max(0, min(J, T - ts));        // its tokens
  const int nb = (nv + LB - 1) / LB;            // its ring blocks
  const int nl = 2 * nb;                        // copies: the fold's, then the replay's
  const size_t row0 = ((size_t)b * T + ts) * C + c;  // (b, ts, c)

  // ---- this warp's ring: the first NS copies go out at once
  auto issue = [&](int n) {
    const int blk = n < nb ? n : n - nb;
    const int s = n % NS;
    unsigned char* st = ring + (size_t)s * kStage;
    mbar_arrive_expect_tx(&bars[s], kStage);
    tma_load_3d(st, &tmk, &bars[s], g * CG, ts + blk * LB, b);
    tma_load_3d(st + kTile * sizeof(KV), &tmv, &bars[s], g * CG, ts + blk * LB, b);
    if (kWT) tma_load_3d(st + 2 * kTile * sizeof(KV), &tmw, &bars[s], g * CG, ts + blk * LB, b);
  };
  int issued = 0;  // lane 0's count of copies issued
  if (lane == 0) {
    if (wp == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (; issued < NS && issued < nl; ++issued) issue(issued);
  }
  __syncwarp();
  bool ok = true;   // every copy this warp waited for arrived in time
  int n = 0;        // copies consumed
  auto wait_copy = [&](int x) {
    const bool got = mbar_wait(&bars[x % NS], (uint32_t)((x / NS) & 1), p.timeout_ns);
    ok = __all_sync(0xffffffffu, got);
    return ok;
  };
  // Stage consumed: its slot takes the next copy. The warp's reads of the
  // stage are ordered before the copy by __syncwarp (the consumer-release /
  // producer-acquire pattern of TMA pipelines; no proxy fence is needed for a
  // read followed by an asynchronous write).
  auto release = [&]() {
    __syncwarp();
    if (lane == 0 && issued < nl) {
      issue(issued);
      ++issued;
    }
  };

  // ---- per-channel constants and the state in
  const float w = (!kWT && cok) ? __ldg(p.w + c) : 0.f;
  const float u = cok ? __ldg(p.u + c) : 0.f;
  Acc xin = acc_empty();
  if (seg == 0 && cok && p.s_num) {
    const size_t i = (size_t)b * C + c;
    xin = acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
  }

  // ---- 1. fold the span, block by block
  Acc agg = acc_empty();
  float wsum = 0.f;
#pragma unroll 1
  for (int blk = 0; blk < nb; ++blk, ++n) {
    if (!wait_copy(n)) break;
    const unsigned char* st = ring + (size_t)(n % NS) * kStage;
    const KV* ks = reinterpret_cast<const KV*>(st) + lane;
    const KV* vs = ks + kTile;
    const int nt = min(LB, nv - blk * LB);
    float kx[LB], vx[LB];
#pragma unroll
    for (int i = 0; i < LB; ++i) {
      kx[i] = Elem<KV>::to_f32(ks[i * CG]);
      vx[i] = Elem<KV>::to_f32(vs[i * CG]);
    }
    if constexpr (kWT) {
      const float* ws = reinterpret_cast<const float*>(st + 2 * kTile * sizeof(KV)) + lane;
      float wx[LB];
#pragma unroll
      for (int i = 0; i < LB; ++i) wx[i] = ws[i * CG];
      float wb;
      const Acc a = nt == LB ? fold_regs_wt<LB>(kx, vx, wx, LB, wb) : fold_regs_wt<LB>(kx, vx, wx, nt, wb);
      agg = combine_wt(agg, a, wb);
      wsum += wb;
    } else if (nt == LB) {
      agg = combine(agg, fold_regs<LB>(kx, vx, LB, w), (float)LB, w);  // (full block: no per-token tests)
    } else {
      agg = combine(agg, fold_regs<LB>(kx, vx, nt, w), (float)nt, w);
    }
    release();
  }
  sagg[wp * CG + lane] = acc_pack(agg);
  if (kWT) swsum[wp * CG + lane] = wsum;
  __syncthreads();

  // ---- 2. prefix of this warp inside the CTA; the last warp forms the total
  Acc pre = acc_empty();
  float wpre = 0.f;  // decay sum of the spans before this warp's (kWT)
  for (int q = 0; q < wp; ++q) {
    const Acc a = acc_unpack(sagg[q * CG + lane]);
    if (kWT) {
      const float wq = swsum[q * CG + lane];
      pre = combine_wt(pre, a, wq);
      wpre += wq;
    } else {
      pre = combine(pre, a, (float)max(0, min(J, T - (t_cta + q * J))), w);
    }
  }
  if (wp == NW - 1) {
    Acc tot;
    float wtot = 0.f;
    if (kWT) {
      tot = combine_wt(pre, agg, wsum);
      wtot = wpre + wsum;
    } else {
      tot = combine(pre, agg, (float)nv, w);
    }
    stot[lane] = acc_pack(tot);
    stotw[lane] = wtot;
  }

  // the totals of the CTAs before this one in the segment, read by warp 0
  // for the whole CTA. Only the warp that wrote this CTA's total releases at
  // the barrier, and in the first segment warp 0, whose read of the state in
  // must come before the state out is written (it may alias); a release in
  // every thread and remote reads in every warp: 364 against 348 us on the
  // long workload, 1 x 65536 x 2048
  if (wp == NW - 1 || (wp == 0 && seg == 0 && p.s_num)) {
    cluster_arrive();
  } else {
    cluster_arrive_relaxed();
  }
  cluster_wait();
  Acc xl = acc_empty();
  float xlw = 0.f;
  if (wp == 0) {
    for (int r = 0; r < rank; ++r) {
      const Acc t = acc_unpack(ld_dsmem_f4(map_shared_rank(&stot[lane], (uint32_t)r)));
      if (kWT) {
        const float wr = ld_dsmem_f32(map_shared_rank(&stotw[lane], (uint32_t)r));
        xl = combine_wt(xl, t, wr);
        xlw += wr;
      } else {
        xl = combine(xl, t, (float)TPC, w);
      }
    }
    sxl[lane] = acc_pack(xl);
    sxw[lane] = xlw;
  }
  // done with the other CTAs' shared memory: warp 0's remote loads have
  // returned (their values are stored above), so no release is needed
  cluster_arrive_relaxed();

  // the segment's incoming state; the last CTA publishes the segment's
  // inclusive prefix for the next segment
  if (wp == 0) {
    if (seg > 0) {
      const uint32_t* flag = p.flags_a + (size_t)(seg - 1) * items + it;
      bool got = ld_acquire_u32(flag) == target;
      if (!got) {
        const uint64_t t0 = global_ns();
        while (!(got = ld_acquire_u32(flag) == target)) {
          if (global_ns() - t0 > p.timeout_ns) break;
          __nanosleep(64);
        }
      }
      got = __all_sync(0xffffffffu, got);
      if (!got && lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
      const size_t islot = ((size_t)(seg - 1) * items + it) * CG + lane;
      sx[lane] = got ? ld_relaxed_f4(p.agg_a + islot) : acc_pack(acc_empty());
    } else {
      sx[lane] = acc_pack(xin);
    }
  }
  __syncthreads();
  const Acc X = acc_unpack(sx[lane]);
  if (wp != 0) {
    xl = acc_unpack(sxl[lane]);
    xlw = sxw[lane];
  }
  if (rank == ncl - 1 && seg < nseg - 1 && wp == 0) {
    // the inclusive prefix of this (full) segment: X, then the CTAs before
    // this one, then this CTA's total
    const Acc own = acc_unpack(stot[lane]);
    Acc incl;
    if (kWT) {
      incl = combine_wt(combine_wt(X, xl, xlw), own, stotw[lane]);
    } else {
      incl = combine(combine(X, xl, (float)(rank * TPC), w), own, (float)TPC, w);
    }
    const size_t oslot = ((size_t)seg * items + it) * CG + lane;
    if (WKV_IN(p.hdr, oslot, (size_t)(nseg - 1) * items * CG)) p.agg_a[oslot] = acc_pack(incl);
    __threadfence();
    __syncwarp();
    // (inject_tile: the test hook that leaves one segment unpublished)
    if (lane == 0 && cl_id != p.inject_tile) st_release_u32(p.flags_a + (size_t)seg * items + it, target);
  }

  // ---- 3. replay the span through the ring (from L2)
  if (ok && nv > 0 && WKV_IN(p.hdr, (size_t)b * T + ts + nv - 1, (size_t)p.B * T)) {
    Acc st;
    float lo = 0.f;
    if (kWT) {
      st = combine_wt(combine_wt(X, xl, xlw), pre, wpre);
    } else {
      st = combine(combine(X, xl, (float)(rank * TPC), w), pre, (float)(wp * J), w);
    }
    OUT* orow = reinterpret_cast<OUT*>(p.out) + row0;
    const KV* rrow = p.r ? reinterpret_cast<const KV*>(p.r) + row0 : nullptr;
    const bool fast = !kWT && __all_sync(0xffffffffu, fast_uw(u, w));
    const float cb[1] = {ex2(fminf(fmaxf(u - w, -kFastUW), kFastUW) * kLog2e)};
    const float w1[1] = {w};
#pragma unroll 1
    for (int blk = 0; blk < nb; ++blk, ++n) {
      if (!wait_copy(n)) break;
      const unsigned char* sb = ring + (size_t)(n % NS) * kStage;
      const KV* ks = reinterpret_cast<const KV*>(sb) + lane;
      const KV* vs = ks + kTile;
      const int nt = min(LB, nv - blk * LB);
      OUT* ob = orow + (size_t)blk * LB * C;
      const KV* rb = rrow ? rrow + (size_t)blk * LB * C : nullptr;
      if (kWT) {
        const float* ws = reinterpret_cast<const float*>(sb + 2 * kTile * sizeof(KV)) + lane;
        for (int i = 0; i < nt; ++i) {
          float o = step_token_wt(st, lo, Elem<KV>::to_f32(ks[i * CG]), Elem<KV>::to_f32(vs[i * CG]), ws[i * CG], u);
          if (rb && cok) o = gate(o, Elem<KV>::to_f32(rb[(size_t)i * C]));
          if (cok) ob[(size_t)i * C] = Elem<OUT>::from_f32(o);
        }
      } else if (fast && nt == LB) {
        // the block's hot loop, compiled once with and once without the gate
        auto run = [&](auto gated) {
          constexpr bool kGate = decltype(gated)::value;
          float kb[LB][1], vb[LB][1], o[LB][1], rg[LB];
          Acc s1[1] = {st};
#pragma unroll
          for (int i = 0; i < LB; ++i) {
            kb[i][0] = Elem<KV>::to_f32(ks[i * CG]);
            vb[i][0] = Elem<KV>::to_f32(vs[i * CG]);
            if (kGate) rg[i] = cok ? Elem<KV>::to_f32(rb[(size_t)i * C]) : 0.f;
          }
          step_tokens<LB, 1>(s1, kb, vb, w1, cb, o);
#pragma unroll
          for (int i = 0; i < LB; ++i) {
            const float oi[1] = {kGate ? gate(o[i][0], rg[i]) : o[i][0]};
            if (cok) stg_stream<OUT, 1>(ob + (size_t)i * C, oi);
          }
          st = s1[0];
        };
        if (rb) {
          run(Flag<true>{});
        } else {
          run(Flag<false>{});
        }
      } else {
        for (int i = 0; i < nt; ++i) {
          const float kk = Elem<KV>::to_f32(ks[i * CG]);
          const float vv = Elem<KV>::to_f32(vs[i * CG]);
          float o = out_token(st, kk, vv, w, u);
          add_token(st, kk, vv, w);
          if (rb && cok) o = gate(o, Elem<KV>::to_f32(rb[(size_t)i * C]));
          if (cok) ob[(size_t)i * C] = Elem<OUT>::from_f32(o);
        }
      }
      release();
    }
    // the warp that holds the last token writes the state out
    if (ok && p.o_num && cok && ts + nv == T && WKV_IN(p.hdr, (size_t)b * C + c, (size_t)p.B * C)) {
      const size_t i = (size_t)b * C + c;
      p.o_num[i] = st.num;
      p.o_den[i] = st.den;
      p.o_max[i] = kWT ? acc_max_e_wt(st, lo) : acc_max_e(st, w);
    }
  }
  if (lane == 0) {
    if (!ok) atomicOr(&p.hdr->status, kStatusWaitTimeout);
    // copies still in flight (after a wait ran out, or a replay that did not
    // run): a bounded chance to land before the CTA leaves
    for (int x = n; x < issued; ++x) (void)mbar_wait(&bars[x % NS], (uint32_t)((x / NS) & 1), p.timeout_ns);
  }
  cluster_wait();
}

}  // namespace wkv
