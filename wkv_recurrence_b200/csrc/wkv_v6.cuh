// The RWKV-v6 matrix-valued state ("RWKV-v6 Architecture: Attention-Free
// Linear Transformers", section "3. Matrix-Valued Hidden State"): per head a
// D x D state S and, per token, d-vectors r_t, w_t, k_t, v_t:
//     S_t = diag(w_t) S_{t-1} + k_t v_t^T,     y_t = sigmoid(r_t) * (S_t k_t).
// Row i of the state evolves on its own (it decays by w_t[i] and gains
// k_t[i] v_t^T) and y_t[i] reads only row i, so the rows are independent
// recurrences: this kernel gives each CTA a block of RB rows of one head and
// walks the sequence, each row's state in registers of NQ threads (8 for
// D >= 64: 8 columns each in fp32 at D = 64), 128 threads per CTA.
//
// Why no tensor cores here: the readout and the update are per-row dot
// products and rank-1 updates with a decay that differs per row, so the only
// dense contractions appear in the chunked reformulation, where the decay is
// folded into the operands (k_s[i] / prod w); in fp32 that needs tf32 or
// bf16 operands on the tensor cores, whose rounding (2^-11 or 2^-9 relative)
// is far above the 1e-5 bar this path is held to, and the ratios of decay
// products overflow fp32 for strong decays. The kernel is bound by its fp32
// instruction issue (3 D^2 fp32 operations per token and head).
//
// Inputs stream through shared memory in blocks of TB tokens (TMA, two stages
// on mbarriers): the block's k and v rows of the head (every row block needs
// all D columns) and the block's r and w for this CTA's rows. Thread q of a
// row owns the 16-byte column chunks q, q+NQ, q+2NQ, ... so that the threads
// of a row read different bank groups, and the rows of a warp read the same
// addresses (broadcast).
#pragma once

#include "wkv_device.cuh"

namespace wkv {

struct V6Params {
  int B, T, H;
  void* y;
  const float* s_in;   // [B, H, D, D] or NULL (zero state)
  float* s_out;        // [B, H, D, D] or NULL; may alias s_in
  WsHeader* hdr;       // status word
  uint64_t timeout_ns;
};

// 2-D tiled TMA load of the box at (x, y) (x the contiguous coordinate).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

template <typename KV, int D, int RB, int TB>
__host__ __device__ constexpr size_t v6_stage_bytes() {
  return (size_t)TB * (2 * D * sizeof(KV) + RB * sizeof(KV) + RB * sizeof(float));
}

// Threads per state row and rows per CTA (128 threads) for head size D: up
// to 8 threads per row, one or more 16-byte column chunks each (measured,
// fp32 D = 64: 171 us with 8 threads of 8 columns against 228 us with 16 of
// 4, whose extra shuffle level and loads outweigh the doubled warp count).
template <typename KV, int D>
struct V6Shape {
  static constexpr int kChunks = D * (int)sizeof(KV) / 16;           // 16-byte chunks per row
  static constexpr int kThreadsPerRow = kChunks < 8 ? kChunks : 8;
  static constexpr int kRows = 128 / kThreadsPerRow;
};

template <typename KV, typename OUT, int D, int RB>
__global__ void __launch_bounds__(128)
    wkv6_fwd(const V6Params p, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
             const __grid_constant__ CUtensorMap tmr, const __grid_constant__ CUtensorMap tmw) {
  constexpr int NQ = V6Shape<KV, D>::kThreadsPerRow;  // threads per row
  static_assert(RB * NQ == 128, "128 threads per CTA");
  constexpr int TB = 32;                       // tokens per staged block
  constexpr int EPC = 16 / sizeof(KV);         // elements per 16-byte chunk
  constexpr int NCH = D / EPC;                 // chunks per row
  constexpr int CPT = NCH / NQ;                // chunks per thread
  constexpr int QD = CPT * EPC;                // columns per thread
  constexpr size_t kStage = v6_stage_bytes<KV, D, RB, TB>();
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 2 * kStage);
  auto sk = [&](int s) { return reinterpret_cast<const KV*>(smem + s * kStage); };
  auto sv = [&](int s) { return reinterpret_cast<const KV*>(smem + s * kStage + TB * D * sizeof(KV)); };
  auto sr = [&](int s) { return reinterpret_cast<const KV*>(smem + s * kStage + 2 * TB * D * sizeof(KV)); };
  auto sw = [&](int s) {
    return reinterpret_cast<const float*>(smem + s * kStage + 2 * TB * D * sizeof(KV) + TB * RB * sizeof(KV));
  };

  const int tid = threadIdx.x;
  const int q = tid & (NQ - 1);
  const int ri = tid / NQ;
  constexpr int NRB = D / RB;
  const int rb = blockIdx.x % NRB;
  const int bh = blockIdx.x / NRB;
  const int h = bh % p.H, b = bh / p.H;
  const int i = rb * RB + ri;  // this thread's row of the state
  const int T = p.T;
  const int row0 = b * T;      // first row of this batch entry in the [B*T, H*D] view
  const int nblk = (T + TB - 1) / TB;

  auto issue = [&](int s, int blk) {
    uint64_t* br = &bar[s];
    unsigned char* base = smem + s * kStage;
    mbar_arrive_expect_tx(br, (uint32_t)kStage);
    tma_load_2d(base, &tmk, br, h * D, row0 + blk * TB);
    tma_load_2d(base + TB * D * sizeof(KV), &tmv, br, h * D, row0 + blk * TB);
    tma_load_2d(base + 2 * TB * D * sizeof(KV), &tmr, br, h * D + rb * RB, row0 + blk * TB);
    tma_load_2d(base + 2 * TB * D * sizeof(KV) + TB * RB * sizeof(KV), &tmw, br, h * D + rb * RB, row0 + blk * TB);
  };
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    issue(0, 0);
    if (nblk > 1) issue(1, 1);
  }

  // this thread's columns: chunks q, q + NQ, ... of the row
  float S[QD];
  const size_t srow = (((size_t)b * p.H + h) * D + i) * D;
#pragma unroll
  for (int m = 0; m < CPT; ++m)
#pragma unroll
    for (int e = 0; e < EPC; ++e) S[m * EPC + e] = p.s_in ? p.s_in[srow + (m * NQ + q) * EPC + e] : 0.f;
  __syncthreads();

  OUT* y = reinterpret_cast<OUT*>(p.y);
  int aborted = -1;
  for (int blk = 0; blk < nblk; ++blk) {
    const int s = blk & 1;
    const bool ok = mbar_wait(&bar[s], (blk >> 1) & 1, p.timeout_ns);
    if (__syncthreads_or(!ok)) {
      aborted = blk;
      break;
    }
    const int nt = min(TB, T - blk * TB);
    const KV* K = sk(s);
    const KV* V = sv(s);
    int tt = 0;
    // full groups of G tokens: the state updates run token after token, but
    // the four-level reductions and gates of the group's outputs overlap
    constexpr int G = 4;
    for (; tt + G <= nt; tt += G) {
      float ki[G], wi[G], rr[G], a[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        ki[j] = Elem<KV>::to_f32(K[(tt + j) * D + i]);
        wi[j] = sw(s)[(tt + j) * RB + ri];
        rr[j] = Elem<KV>::to_f32(sr(s)[(tt + j) * RB + ri]);
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < CPT; ++m) {
          float kv[EPC], vv[EPC];
          load_vec<KV, EPC>(K + (tt + j) * D + (m * NQ + q) * EPC, kv);
          load_vec<KV, EPC>(V + (tt + j) * D + (m * NQ + q) * EPC, vv);
#pragma unroll
          for (int e = 0; e < EPC; ++e) {
            float& x = S[m * EPC + e];
            x = fmaf(wi[j], x, ki[j] * vv[e]);
            acc[e & 3] = fmaf(x, kv[e], acc[e & 3]);
          }
        }
        a[j] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      }
#pragma unroll
      for (int o = 1; o < NQ; o <<= 1)
#pragma unroll
        for (int j = 0; j < G; ++j) a[j] += __shfl_xor_sync(0xffffffffu, a[j], o);
      if (q == 0) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const size_t yi = (((size_t)row0 + blk * TB + tt + j) * p.H + h) * D + i;
          if (WKV_IN(p.hdr, yi, (size_t)p.B * T * p.H * D)) y[yi] = Elem<OUT>::from_f32(gate(a[j], rr[j]));
        }
      }
    }
    for (; tt < nt; ++tt) {
      const float ki = Elem<KV>::to_f32(K[tt * D + i]);
      const float wi = sw(s)[tt * RB + ri];
      const float rr = Elem<KV>::to_f32(sr(s)[tt * RB + ri]);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < CPT; ++m) {
        float kv[EPC], vv[EPC];
        load_vec<KV, EPC>(K + tt * D + (m * NQ + q) * EPC, kv);
        load_vec<KV, EPC>(V + tt * D + (m * NQ + q) * EPC, vv);
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          float& x = S[m * EPC + e];
          x = fmaf(wi, x, ki * vv[e]);
          acc[e & 3] = fmaf(x, kv[e], acc[e & 3]);
        }
      }
      float a = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
      for (int o = 1; o < NQ; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      const size_t yi = (((size_t)row0 + blk * TB + tt) * p.H + h) * D + i;
      if (q == 0 && WKV_IN(p.hdr, yi, (size_t)p.B * T * p.H * D)) y[yi] = Elem<OUT>::from_f32(gate(a, rr));
    }
    __syncthreads();  // every thread is done with stage s
    if (tid == 0 && blk + 2 < nblk) {
      fence_proxy_async_smem();
      issue(s, blk + 2);
    }
  }
  if (aborted >= 0) {
    if (tid == 0) {
      atomicOr(&p.hdr->status, kStatusWaitTimeout);
      for (int x = aborted; x < nblk && x < aborted + 2; ++x) (void)mbar_wait(&bar[x & 1], (x >> 1) & 1, p.timeout_ns);
    }
    return;
  }
  if (p.s_out && WKV_IN(p.hdr, srow + D - 1, (size_t)p.B * p.H * D * D)) {
#pragma unroll
    for (int m = 0; m < CPT; ++m)
#pragma unroll
      for (int e = 0; e < EPC; ++e) p.s_out[srow + (m * NQ + q) * EPC + e] = S[m * EPC + e];
  }
}

}  // namespace wkv
