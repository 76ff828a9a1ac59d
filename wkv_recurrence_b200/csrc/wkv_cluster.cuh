// The chunked scan over T in one thread-block cluster: for sequences short
// enough that one cluster's shared memory holds all of a channel group's k and
// v (T <= 8 CTAs x NW*J tokens), there is no chunk total in global memory, no
// look-back between CTAs and no second read of the inputs.
//
// One cluster of ncl CTAs takes one (batch row, 32-channel group) and the
// whole sequence; CTA `rank` of the cluster holds tokens
// [rank*TPC, (rank+1)*TPC) (TPC = NW*J) in shared memory, one span of J tokens
// per warp, one channel per lane:
//   1. each warp copies its span of k and v in (TMA, one mbarrier per span) and
//      folds it from the empty state into an aggregate (largest end-of-span
//      exponent first, then the weighted sums);
//   2. each warp combines the aggregates of the warps before it (its prefix
//      inside the CTA); the last warp also forms the CTA's total;
//   3. after a cluster barrier, every CTA reads the totals of the CTAs before
//      it from their shared memory (distributed shared memory) and combines
//      them in order, starting from the state in: its incoming state;
//   4. each warp replays its span from (incoming state + prefix) out of shared
//      memory and writes the outputs (gated by sigmoid(r) when r is given);
//      the warp that holds token T-1 writes the state out.
// The order of every combine depends on the shape only (results are bitwise
// reproducible). With kWT the decay is per token ("RWKV-v6 Architecture",
// section "2. Dynamic Data-Dependent Decay"): w_t comes in as a third tile and
// the combines carry each span's decay sum.
//
// Every CTA reads the state in before the first cluster barrier and the state
// out is written after it, so state_out may alias state_in. A second cluster
// barrier (arrive after the last remote read, wait before exit) keeps every
// CTA's shared memory alive while others may read it. All threads of every CTA
// take both barriers; no thread returns early.
#pragma once

#include "wkv_device.cuh"
#include "wkv_fwd.cuh"

namespace wkv {

// Shared-memory bytes of wkv_fwd_cluster.
template <typename KV, int NW, int J, bool kWT>
__host__ __device__ constexpr size_t cluster_smem_bytes() {
  return (size_t)NW * J * 32 * (2 * sizeof(KV) + (kWT ? 4 : 0))  // k, v (and w_t) tiles
         + (size_t)NW * 32 * (16 + (kWT ? 4 : 0))                 // span aggregates (and decay sums)
         + 32 * (16 + 4)                                          // the CTA's total and decay sum
         + (size_t)NW * 8;                                        // one mbarrier per span
}

template <typename KV, typename OUT, int NW, int J, bool kWT>
__global__ void __launch_bounds__(NW * 32)
    wkv_fwd_cluster(const FwdParams p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmw) {
  constexpr int CG = 32;
  constexpr int TPC = NW * J;
  constexpr int kSpan = J * CG;  // elements of one tensor in one span
  constexpr uint32_t kSpanBytes = (uint32_t)(2 * kSpan * sizeof(KV) + (kWT ? kSpan * 4 : 0));
  extern __shared__ __align__(1024) unsigned char smem[];
  KV* ktile = reinterpret_cast<KV*>(smem);  // [TPC][CG]
  KV* vtile = ktile + TPC * CG;             // [TPC][CG]
  float* wtile = reinterpret_cast<float*>(vtile + TPC * CG);                                   // [TPC][CG] (kWT)
  float4* sagg = reinterpret_cast<float4*>(wtile + (kWT ? TPC * CG : 0));                      // [NW][CG]
  float* swsum = reinterpret_cast<float*>(sagg + NW * CG);                                     // [NW][CG] (kWT)
  float4* stot = reinterpret_cast<float4*>(swsum + (kWT ? NW * CG : 0));                       // [CG]
  float* stotw = reinterpret_cast<float*>(stot + CG);                                          // [CG]
  uint64_t* bar = reinterpret_cast<uint64_t*>(stotw + CG);                                     // [NW]

  const int lane = threadIdx.x & 31;
  const int wp = threadIdx.x >> 5;
  const int T = p.T, C = p.C;
  const int ncl = p.cluster;
  const int rank = (int)(blockIdx.x % (unsigned)ncl);
  const int item = (int)(blockIdx.x / (unsigned)ncl);
  const int ngc = (C + CG - 1) / CG;
  const int b = item / ngc, g = item % ngc;
  const int c = g * CG + lane;
  const bool cok = c < C;
  const int t_cta = rank * TPC;
  const int ts = t_cta + wp * J;
  const int nv = max(0, min(J, T - ts));

  // ---- copy this warp's span in
  KV* ks = ktile + wp * kSpan + lane;
  KV* vs = vtile + wp * kSpan + lane;
  float* wsp = wtile + wp * kSpan + lane;
  if (lane == 0 && nv > 0) {
    mbar_init(&bar[wp], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar[wp], kSpanBytes);
    tma_load_3d(ktile + wp * kSpan, &tmk, &bar[wp], g * CG, ts, b);
    tma_load_3d(vtile + wp * kSpan, &tmv, &bar[wp], g * CG, ts, b);
    if (kWT) tma_load_3d(wtile + wp * kSpan, &tmw, &bar[wp], g * CG, ts, b);
  }
  __syncwarp();

  // ---- per-channel constants and the state in (read before the first
  // cluster barrier: state_out may alias it)
  const float w = (!kWT && cok) ? __ldg(p.w + c) : 0.f;
  const float u = cok ? __ldg(p.u + c) : 0.f;
  Acc xin = acc_empty();
  if (cok && p.s_num) {
    const size_t i = (size_t)b * C + c;
    xin = acc_from_state(p.s_num[i], p.s_den[i], p.s_max[i]);
  }

  // ---- 1. fold the span
  bool copy_ok = true;
  Acc agg = acc_empty();
  float wsum = 0.f;
  if (nv > 0) {
    copy_ok = mbar_wait(&bar[wp], 0, p.timeout_ns);
    if (!copy_ok) {
      if (lane == 0) atomicOr(&p.hdr->status, kStatusWaitTimeout);
    } else if (kWT) {
      Acc a1[1];
      float s1[1];
      aggregate_span_wt<KV, J, 1, CG>(ks, vs, wsp, nv, a1, s1);
      agg = a1[0];
      wsum = s1[0];
    } else {
      Acc a1[1];
      const float w1[1] = {w};
      aggregate_tile_span<KV, J, 1, CG>(ks, vs, nv, w1, a1);
      agg = a1[0];
    }
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

  // ---- 3. incoming state of this CTA from the totals of the CTAs before it
  cluster_arrive();
  cluster_wait();
  Acc x = xin;
  for (int r = 0; r < rank; ++r) {
    const Acc t = acc_unpack(ld_dsmem_f4(map_shared_rank(&stot[lane], (uint32_t)r)));
    if (kWT) {
      x = combine_wt(x, t, ld_dsmem_f32(map_shared_rank(&stotw[lane], (uint32_t)r)));
    } else {
      x = combine(x, t, (float)TPC, w);
    }
  }
  cluster_arrive();  // done with the other CTAs' shared memory

  // ---- 4. replay the span
  if (nv > 0 && copy_ok && WKV_IN(p.hdr, (size_t)b * T + ts + nv - 1, (size_t)p.B * T)) {
    Acc st = kWT ? combine_wt(x, pre, wpre) : combine(x, pre, (float)(wp * J), w);
    OUT* orow = reinterpret_cast<OUT*>(p.out) + ((size_t)b * T + ts) * C + c;
    const KV* rrow = p.r ? reinterpret_cast<const KV*>(p.r) + ((size_t)b * T + ts) * C + c : nullptr;
    float lo = 0.f;
    if (kWT) {
      for (int i = 0; i < nv; ++i) {
        float kx[1], vx[1];
        load_vec<KV, 1>(ks + i * CG, kx);
        load_vec<KV, 1>(vs + i * CG, vx);
        float o = step_token_wt(st, lo, kx[0], vx[0], wsp[i * CG], u);
        if (rrow) o = gate(o, Elem<KV>::to_f32(rrow[(size_t)i * C]));
        if (cok) orow[(size_t)i * C] = Elem<OUT>::from_f32(o);
      }
    } else {
      const bool fast = __all_sync(0xffffffffu, fast_uw(u, w));
      const float cb[1] = {ex2(fminf(fmaxf(u - w, -kFastUW), kFastUW) * kLog2e)};
      const float w1[1] = {w};
      Acc s1[1] = {st};
      if (fast && nv == J) {
        // the span's hot loop, compiled once with and once without the gate
        auto span = [&](auto gated) {
          constexpr bool kGate = decltype(gated)::value;
          constexpr int NB = J < 8 ? J : 8;
#pragma unroll
          for (int j0 = 0; j0 < J; j0 += NB) {
            float kb[NB][1], vb[NB][1], ob[NB][1], rb[NB];
#pragma unroll
            for (int jj = 0; jj < NB; ++jj) {
              load_vec<KV, 1>(ks + (j0 + jj) * CG, kb[jj]);
              load_vec<KV, 1>(vs + (j0 + jj) * CG, vb[jj]);
              if (kGate) rb[jj] = Elem<KV>::to_f32(rrow[(size_t)(j0 + jj) * C]);
            }
            step_tokens<NB, 1>(s1, kb, vb, w1, cb, ob);
#pragma unroll
            for (int jj = 0; jj < NB; ++jj) {
              const float o = kGate ? gate(ob[jj][0], rb[jj]) : ob[jj][0];
              if (cok) orow[(size_t)(j0 + jj) * C] = Elem<OUT>::from_f32(o);
            }
          }
        };
        if (rrow) {
          span(Flag<true>{});
        } else {
          span(Flag<false>{});
        }
      } else {
        for (int i = 0; i < nv; ++i) {
          float kx[1], vx[1];
          load_vec<KV, 1>(ks + i * CG, kx);
          load_vec<KV, 1>(vs + i * CG, vx);
          float o = out_token(s1[0], kx[0], vx[0], w, u);
          add_token(s1[0], kx[0], vx[0], w);
          if (rrow) o = gate(o, Elem<KV>::to_f32(rrow[(size_t)i * C]));
          if (cok) orow[(size_t)i * C] = Elem<OUT>::from_f32(o);
        }
      }
      st = s1[0];
    }
    // the warp that holds the last token writes the state out
    if (p.o_num && cok && ts + nv == T && WKV_IN(p.hdr, (size_t)b * C + c, (size_t)p.B * C)) {
      const size_t i = (size_t)b * C + c;
      p.o_num[i] = st.num;
      p.o_den[i] = st.den;
      p.o_max[i] = kWT ? acc_max_e_wt(st, lo) : acc_max_e(st, w);
    }
  }
  if (nv > 0 && !copy_ok && lane == 0) (void)mbar_wait(&bar[wp], 0, p.timeout_ns);  // bounded drain
  cluster_wait();
}

}  // namespace wkv
