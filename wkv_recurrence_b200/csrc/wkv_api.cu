// C ABI of libwkv.so (declared in include/wkv.h): argument checks, the choice
// of kernel and tile sizes, workspace layout, TMA descriptors and launches.
// Nothing here allocates device memory; the caller passes every buffer.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/wkv.h"
#include "wkv_bwd.cuh"
#include "wkv_cluster.cuh"
#include "wkv_device.cuh"
#include "wkv_fwd.cuh"
#include "wkv_step.cuh"
#include "wkv_v6.cuh"

namespace wkv {
namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;  // 1 s

// ---------------------------------------------------------------------------
// kernel configurations
// ---------------------------------------------------------------------------
// sequential kernel: CTA = 32, 64 or 128 threads x VEC channels, LT-token tiles
// (tokens per stage for 2 channels per thread; twice as many for 1)
constexpr int kSeqLtF32 = 8, kSeqStagesF32 = 4;    // 4 stages of 64 B x CG
constexpr int kSeqLtBf16 = 16, kSeqStagesBf16 = 4;  // 4 stages of 64 B x CG
constexpr int kSeqFallbackVec = 1, kSeqFallbackLt = 16;

// chunked kernel: a tile is 64 channels (32 lanes x 2) by L = NW x 16 tokens
constexpr int kChunkRW = 32, kChunkVec = 2, kChunkCG = kChunkRW * kChunkVec;
// the automatic choice gives the sequential kernel one channel per thread below
// this many channels (148 SMs x 16 warps x 64 channels)
constexpr long long kSeqVec1MaxLanes = 148ll * 16 * 64;
// Above this many elements of k (and as many of v: 128 MiB of both in fp32,
// about the size of L2) the automatic choice for few channels is the cluster
// scan, which reads k and v from HBM once, instead of the three-launch scan,
// whose second read of k and v hits L2 only while they fit there (layer,
// 8 x 1024 x 768: 23.5 us three-launch against 25.0 cluster; long,
// 1 x 65536 x 2048: 426 against 364 us; the same at T = 16384: 114 against
// 104 us).
constexpr long long kClusterMinElems = 1ll << 24;

struct Plan {
  int kernel;  // 1 seq, 2 chunked single launch, 3 chunked in three launches, 4 pipelined chunked, 5 cluster
  int cw;      // cluster scan: warps (spans) per CTA
  int cj;      // cluster scan: tokens per span
  int ncl;     // cluster scan: CTAs per cluster
  int nseg;    // cluster scan: segments (clusters) per (batch row, 32-channel group)
  int seq_threads;  // CTA width of the sequential kernel
  int seq_vec;      // channels per thread of the sequential kernel
  int scan_segments;  // three-launch scan: segments per channel in the scan of chunk totals
  int replay_chunks;  // three-launch scan: consecutive chunks per replay CTA
  int replay_threads;  // three-launch scan: threads (channels) per replay CTA
  int stages;       // pipelined chunked scan: ring stages (0 = choose at launch)
  int L;       // chunk length (chunk kernel)
  int J;       // tokens per warp (chunk kernel)
  int G;       // look-back group
  int NG;      // channel groups per batch row
  int nch;     // chunks per sequence
  long long n_tiles;
  long long nblk;  // look-back groups per sequence
  size_t off_flags_a, off_flags_p, off_agg_a, off_agg_p, off_x0, off_wtot, bytes;
};


// The last CUDA error this library met in the calling thread (for
// wkv_last_cuda_error), recorded wherever a call returns WKV_ERR_CUDA because
// of one.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

bool cuda_ok(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = e;
  return e == cudaSuccess;
}

// Status of the launch just made (<<<>>> launches report only through
// cudaGetLastError).
wkv_status launch_result() { return cuda_ok(cudaGetLastError()) ? WKV_OK : WKV_ERR_CUDA; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The plan for a call: which kernel, tile sizes, and the workspace layout.
// tma_ok = false (inputs that TMA cannot address: misaligned base, row pitch
// not a multiple of 16 bytes) turns the three-launch, pipelined and cluster
// scans, which need TMA, into the single-launch one (the sequential kernel
// with per-token decays; the pipelined scan uses the same workspace layout as
// the single-launch one). Three-launch and cluster plans reserve enough
// workspace for the fallback, so a workspace sized by
// wkv_forward_workspace_size always fits.
bool make_plan(int64_t B, int64_t T, int64_t C, const wkv_options* o, Plan* pl, bool tma_ok = true,
               bool wt = false) {
  std::memset(pl, 0, sizeof *pl);
  const int want = o ? o->kernel : 0;
  if (want < 0 || want > 5) return false;
  const int64_t lanes = B * C;
  // the cluster scan's CTA shape: cw spans of cj tokens per CTA, up to
  // kClusterMaxCTAs CTAs per cluster and segment
  if (o && o->cta_warps != 0 && o->cta_warps != 4 && o->cta_warps != 8) return false;
  const int cw = (o && o->cta_warps) ? o->cta_warps : 8;
  const int cj = (want == 5 && o && o->span) ? o->span : 64;
  if (cj != 32 && cj != 64) return false;
  int kernel = want;
  if (kernel == 0) {
    if (lanes >= 65536 || T <= 64) {
      kernel = 1;
    } else if (lanes * T > kClusterMinElems) {
      kernel = 5;  // k and v larger than L2: read them once
    } else {
      kernel = 3;  // the three-launch scan (its second read of k and v hits L2)
    }
  }
  // per-token decays: the sequential, three-launch and cluster kernels only
  if (wt && (kernel == 2 || kernel == 4)) return false;
  const bool three_requested = (kernel == 3);
  if ((kernel == 3 || kernel == 4 || kernel == 5) && !tma_ok) kernel = wt ? 1 : 2;
  pl->kernel = kernel;
  pl->cw = cw;
  pl->cj = cj;
  {
    const int64_t tpc = (int64_t)cw * cj;
    pl->ncl = (int)std::min<int64_t>(kClusterMaxCTAs, std::max<int64_t>(1, (T + tpc - 1) / tpc));
    const int64_t seg_tokens = pl->ncl * tpc;
    pl->nseg = (int)std::max<int64_t>(1, (T + seg_tokens - 1) / seg_tokens);
  }
  pl->bytes = sizeof(WsHeader);
  if (o && o->scan_segments != 0 && o->scan_segments != 1 && o->scan_segments != 4 && o->scan_segments != 16 &&
      o->scan_segments != 64)
    return false;
  if (o && (o->stages < 0 || o->stages == 1 || o->stages > 8)) return false;
  if (o && (o->seq_vec < 0 || o->seq_vec > 2)) return false;
  if (o && o->replay_chunks != 0 && o->replay_chunks != 1 && o->replay_chunks != 2 && o->replay_chunks != 4)
    return false;
  pl->replay_chunks = (o && o->replay_chunks) ? o->replay_chunks : 1;
  // one channel per thread doubles the warps of the sequential kernel; worth
  // it while two per thread would leave fewer than ~16 warps per SM (measured,
  // 65536 channels: 377 vs 424 us)
  pl->seq_vec = (o && o->seq_vec) ? o->seq_vec : (lanes < kSeqVec1MaxLanes ? 1 : 2);
  pl->stages = o ? o->stages : 0;
  pl->scan_segments = o ? o->scan_segments : 0;
  int sth = o ? o->seq_threads : 0;
  if (sth == 0) sth = 32;  // many small CTAs: more resident warps per SM
  if (sth != 32 && sth != 64 && sth != 128) return false;
  pl->seq_threads = sth;
  if (kernel == 1) return true;
  if (kernel == 5) {
    // one segment: the header only; more: a flag and an inclusive prefix
    // (32 float4) per (segment but the last, batch row, 32-channel group)
    const int64_t items = B * ((C + 31) / 32);
    if ((int64_t)pl->nseg * items * pl->ncl >= (1ll << 31)) return false;
    size_t off = sizeof(WsHeader);
    pl->off_flags_a = off;
    off = round_up(off + sizeof(uint32_t) * (size_t)(pl->nseg - 1) * items, 256);
    pl->off_agg_a = off;
    off = round_up(off + sizeof(float4) * (size_t)(pl->nseg - 1) * items * 32, 256);
    pl->bytes = pl->nseg > 1 ? off : sizeof(WsHeader);
    // a call whose inputs TMA cannot address runs the single-launch scan (or,
    // with per-token decays, the sequential kernel) instead: reserve for it too
    wkv_options o2;
    if (o) {
      o2 = *o;
    } else {
      std::memset(&o2, 0, sizeof o2);
    }
    o2.kernel = wt ? 1 : 2;
    o2.cta_warps = 0;
    o2.span = 0;
    Plan p2;
    if (!make_plan(B, T, C, &o2, &p2, false, wt)) return false;
    pl->bytes = std::max(pl->bytes, p2.bytes);
    return true;
  }

  int L = o ? o->chunk_len : 0;
  if (L == 0) {
    // the three-launch scan replays every (batch row, chunk, 32 channels) as
    // one warp: 32-token chunks where 64-token ones would give fewer than 8192
    // such warps (measured, layer: 25.3 vs 26.5 us), else 64 (long: 424 us at
    // both 64 and 128, 440 at 32)
    if (kernel == 3) {
      L = (B * C * ((T + 63) / 64)) / 32 < 8192 ? 32 : 64;
    } else {
      L = 128;
    }
  }
  if (L != 32 && L != 64 && L != 128) return false;
  int J = o ? o->span : 0;
  if (J == 0) J = 16;
  if (J != 8 && J != 16) return false;
  if (wt && kernel == 3 && J != 16) return false;  // per-token decays: 16-token spans
  // the pipelined scan runs L/J fold and L/J replay warps plus two: at most 8
  // of each keeps the CTA within 1024 threads
  if (kernel == 4 && L / J > 8) return false;
  int G = o ? o->lookback_group : 0;
  if (G == 0) G = 16;
  if (G < 1 || G > 1024) return false;
  pl->L = L;
  pl->J = J;
  pl->G = G;
  pl->NG = (int)((C + kChunkCG - 1) / kChunkCG);
  pl->nch = (int)((T + L - 1) / L);
  // the replay pass: 32 channels per CTA unless asked otherwise (the most
  // resident warps; layer: 23.8 us against 24.2 and 24.7 at 64 and 128; long:
  // within 1.5% at all three)
  pl->replay_threads = (o && o->seq_threads) ? o->seq_threads : 32;
  const long long BNG = (long long)B * pl->NG;
  pl->n_tiles = (long long)pl->nch * BNG;
  if (pl->n_tiles >= (1ll << 31)) return false;
  pl->nblk = (pl->nch + G - 1) / G;
  // three-launch layout: totals of all chunks but the last, incoming states
  // of all chunks
  size_t off3 = sizeof(WsHeader);
  const size_t t_tot = off3;
  off3 = round_up(off3 + sizeof(float4) * (size_t)(std::max(pl->nch - 1, 0) * BNG) * kChunkCG, 256);
  const size_t t_x0 = off3;
  off3 = round_up(off3 + sizeof(float4) * (size_t)pl->n_tiles * kChunkCG, 256);
  // with per-token decays, the decay sum of each chunk total
  const size_t t_w = off3;
  off3 = round_up(off3 + sizeof(float) * (size_t)(std::max(pl->nch - 1, 0) * BNG) * kChunkCG, 256);
  // single-launch layout: flags, chunk totals, group prefixes
  size_t off = sizeof(WsHeader);
  pl->off_flags_a = off;
  off = round_up(off + sizeof(uint32_t) * (size_t)pl->n_tiles, 256);
  pl->off_flags_p = off;
  off = round_up(off + sizeof(uint32_t) * (size_t)(pl->nblk * BNG), 256);
  pl->off_agg_a = off;
  off = round_up(off + sizeof(float4) * (size_t)pl->n_tiles * kChunkCG, 256);
  pl->off_agg_p = off;
  off = round_up(off + sizeof(float4) * (size_t)(pl->nblk * BNG) * kChunkCG, 256);
  if (kernel == 3) {
    pl->off_flags_a = pl->off_flags_p = pl->off_agg_p = 0;
    pl->off_agg_a = t_tot;
    pl->off_x0 = t_x0;
    pl->off_wtot = t_w;
    pl->bytes = std::max(off3, off);
  } else {
    pl->bytes = three_requested ? std::max(off3, off) : off;
  }
  return true;
}

// Sizes wkv_forward accepts: B, T, C >= 0, T < 2^24, B and C < 2^31 and
// B*T*C < 2^62 (checked without overflow).
bool sizes_ok(int64_t B, int64_t T, int64_t C) {
  if (B < 0 || T < 0 || C < 0) return false;
  if (T >= (1ll << 24) || C >= (1ll << 31) || B >= (1ll << 31)) return false;
  if (B > 0 && C > 0 && T > (int64_t)((1ull << 62) / (uint64_t)(B * C))) return false;
  return true;
}

// Every check of wkv_forward's arguments that needs no plan and no workspace:
// sizes, dtypes, state structs, options, and the pointers the sizes require.
wkv_status check_forward_args(int64_t B, int64_t T, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype,
                              const float* w, const float* u, const void* out, wkv_dtype out_dtype,
                              const wkv_cstate* state_in, const wkv_state* state_out, const wkv_options* opts) {
  if (!sizes_ok(B, T, C)) return WKV_ERR_INVALID_ARG;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (out_dtype != WKV_F32 && out_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (kv_dtype == WKV_F32 && out_dtype != WKV_F32) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (state_in && (!state_in->num || !state_in->den || !state_in->max_e)) return WKV_ERR_INVALID_ARG;
  if (state_out && (!state_out->num || !state_out->den || !state_out->max_e)) return WKV_ERR_INVALID_ARG;
  if (opts && opts->wait_timeout_ns < 0) return WKV_ERR_INVALID_ARG;
  if (opts && (opts->inject_enable != 0 && opts->inject_enable != 1)) return WKV_ERR_INVALID_ARG;
  if (B * T * C > 0 && (!k || !v || !out)) return WKV_ERR_INVALID_ARG;
  if (B * C > 0 && T > 0 && (!w || !u)) return WKV_ERR_INVALID_ARG;
  return WKV_OK;
}

bool tma_usable(const void* k, const void* v, int64_t C, size_t es) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(k), b = reinterpret_cast<uintptr_t>(v);
  return a % 16 == 0 && b % 16 == 0 && (C * (int64_t)es) % 16 == 0;
}

// ---------------------------------------------------------------------------
// device facts and per-kernel setup, cached per device
// ---------------------------------------------------------------------------
struct DevInfo {
  int sms = 0;
  int smem_optin = 0;
};
std::mutex g_mu;
DevInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices];

bool dev_info(int dev, DevInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev_ok[dev]) {
    DevInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return false;
    g_dev[dev] = d;
    g_dev_ok[dev] = true;
  }
  *out = g_dev[dev];
  return true;
}

// Raises the dynamic shared memory limit of kernel `fn` on device `dev` to at
// least `smem` and returns how many CTAs of it fit on one SM with that much
// shared memory. The limit is an attribute of the kernel, shared by every
// launch of it, so it only ever grows (a launch with less shared memory must
// not lower it under a later, larger one); occupancies are cached per size.
struct KernelSetup {
  const void* fn;
  int dev;
  size_t smem;
  int occ;
};
struct KernelLimit {
  const void* fn;
  int dev;
  size_t smem;
};
std::vector<KernelSetup> g_setups;
std::vector<KernelLimit> g_limits;

template <typename F>
bool kernel_setup(F fn, int dev, int threads, size_t smem, int* blocks_per_sm) {
  const void* key = reinterpret_cast<const void*>(fn);
  std::lock_guard<std::mutex> lk(g_mu);
  KernelLimit* lim = nullptr;
  for (KernelLimit& l : g_limits)
    if (l.fn == key && l.dev == dev) lim = &l;
  if (!lim || lim->smem < smem) {
    if (!cuda_ok(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))) return false;
    if (lim) {
      lim->smem = smem;
    } else {
      g_limits.push_back(KernelLimit{key, dev, smem});
    }
  }
  for (const KernelSetup& s : g_setups) {
    if (s.fn == key && s.dev == dev && s.smem == smem) {
      *blocks_per_sm = s.occ;
      return true;
    }
  }
  int n = 0;
  if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem))) return false;
  g_setups.push_back(KernelSetup{key, dev, smem, n});
  *blocks_per_sm = n;
  return true;
}

// ---------------------------------------------------------------------------
// TMA descriptors
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, T, C] tensor, box [1, rows, cols] (cols contiguous)
bool make_tmap(CUtensorMap* m, const void* base, wkv_dtype dt, int64_t B, int64_t T, int64_t C, int rows, int cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const size_t es = dt == WKV_F32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)(C * es), (cuuint64_t)(T * C * es)};
  cuuint32_t box[3] = {(cuuint32_t)cols, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt == WKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename KV, typename OUT, int THREADS, int VEC, int LT, int STAGES, bool kTMA, bool kWT = false>
wkv_status launch_seq(const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tw,
                      cudaStream_t st, int dev) {
  constexpr int CG = THREADS * VEC;
  const size_t smem = (size_t)STAGES * seq_stage_bytes<KV, LT, CG, kWT>() + 64 * STAGES;
  auto fn = wkv_fwd_seq<KV, OUT, VEC, THREADS, LT, STAGES, kTMA, false, kWT>;
  int occ = 0;
  if (!kernel_setup(fn, dev, THREADS, smem, &occ)) return WKV_ERR_CUDA;
  FwdParams q = p;
  q.NG = (p.C + CG - 1) / CG;
  const long long grid = (long long)p.B * q.NG;
  if (grid >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  fn<<<(unsigned)grid, THREADS, smem, st>>>(q, tk, tv, tw);
  return launch_result();
}

template <typename KV, typename OUT, int NW, int J, bool kTMA>
wkv_status launch_chunk(const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st, int dev) {
  if (!p.flags_a || !p.flags_p || !p.agg_a || !p.agg_p || !p.hdr) return WKV_ERR_INVALID_ARG;
  constexpr int L = NW * J;
  const size_t smem = 2ull * L * kChunkCG * sizeof(KV) + sizeof(float4) * (NW + 1) * kChunkCG + 64;
  auto fn = wkv_fwd_chunk<KV, OUT, NW, J, kTMA>;
  int occ = 0;
  if (!kernel_setup(fn, dev, (NW + 1) * 32, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  fn<<<(unsigned)p.n_tiles, (NW + 1) * 32, smem, st>>>(p, tk, tv);
  return launch_result();
}

// Persistent launch of the pipelined chunked scan: as many CTAs as fit on the
// device at once (never more than there are tiles). `stages` = 0 chooses the
// deepest ring of up to 8 stages that fits in one CTA's shared memory.
template <typename KV, typename OUT, int NC, int J>
wkv_status launch_pipe(const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st, int dev,
                       const DevInfo& di, int stages) {
  if (!p.flags_a || !p.flags_p || !p.agg_a || !p.agg_p || !p.hdr) return WKV_ERR_INVALID_ARG;
  constexpr size_t kStage = 2ull * NC * J * kChunkCG * sizeof(KV);
  auto bytes = [](int s) { return (size_t)s * kStage + pipe_aux_bytes<NC>(s); };
  if (stages == 0) {
    stages = 8;
    while (stages > 2 && bytes(stages) > (size_t)di.smem_optin) --stages;
  }
  const size_t smem = bytes(stages);
  if (smem > (size_t)di.smem_optin) return WKV_ERR_INVALID_ARG;
  auto fn = wkv_fwd_pipe<KV, OUT, NC, J>;
  int occ = 0;
  if (!kernel_setup(fn, dev, (2 * NC + 2) * 32, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  FwdParams q = p;
  q.stages = stages;
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>((long long)occ * di.sms, p.n_tiles));
  fn<<<grid, (2 * NC + 2) * 32, smem, st>>>(q, tk, tv);
  return launch_result();
}

template <typename KV, typename OUT>
wkv_status launch_pipe_shape(const Plan& pl, const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                             cudaStream_t st, int dev, const DevInfo& di) {
  if (pl.J == 8) {  // make_plan refuses L = 128 with J = 8 for this kernel
    if (pl.L == 32) return launch_pipe<KV, OUT, 4, 8>(p, tk, tv, st, dev, di, pl.stages);
    return launch_pipe<KV, OUT, 8, 8>(p, tk, tv, st, dev, di, pl.stages);
  }
  switch (pl.L) {
    case 32: return launch_pipe<KV, OUT, 2, 16>(p, tk, tv, st, dev, di, pl.stages);
    case 64: return launch_pipe<KV, OUT, 4, 16>(p, tk, tv, st, dev, di, pl.stages);
    default: return launch_pipe<KV, OUT, 8, 16>(p, tk, tv, st, dev, di, pl.stages);
  }
}

// Launch configuration with programmatic stream serialization: the launch may
// begin while the previous one on the stream drains; the kernel orders itself
// with griddepcontrol.
struct PdlConfig {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  PdlConfig(dim3 grid, dim3 block, size_t smem, cudaStream_t st) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};

// The three-launch chunked scan: chunk totals (A), their scan (S), the replay
// (B, launched with programmatic stream serialization so that its tile copies
// overlap the scan).
// The replay pass of the three-launch scan: the sequential kernel in chunked
// mode, one warp per (batch row, chunk, 32 channels), launched with
// programmatic stream serialization after the scan.
template <typename KV, typename OUT, int TH, int LT, int STAGES, bool kWT = false>
wkv_status launch_seq_chunks(const FwdParams& p, const CUtensorMap& bk, const CUtensorMap& bv, cudaStream_t st,
                             int dev, const CUtensorMap* bw = nullptr) {
  auto fb = wkv_fwd_seq<KV, OUT, 1, TH, LT, STAGES, true, true, kWT>;
  const size_t smem = (size_t)STAGES * seq_stage_bytes<KV, LT, TH, kWT>() + 64 * STAGES;
  int occ = 0;
  if (!kernel_setup(fb, dev, TH, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  const long long nseq = (p.nch + p.replay_chunks - 1) / p.replay_chunks;
  const long long grid = (long long)p.B * nseq * ((p.C + TH - 1) / TH);
  if (grid >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  PdlConfig cb(dim3((unsigned)grid), dim3(TH), smem, st);
  if (!cuda_ok(cudaLaunchKernelEx(&cb.cfg, fb, p, bk, bv, bw ? *bw : bv))) return WKV_ERR_CUDA;
  return launch_result();
}

template <typename KV, typename OUT, int NW, int J, bool kWT>
wkv_status launch_tile3(const Plan& pl, const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                        wkv_dtype kvdt, cudaStream_t st, int dev) {
  if (!p.agg_a || !p.x0 || !p.hdr || (kWT && !p.wtot)) return WKV_ERR_INVALID_ARG;
  constexpr int L = NW * J;
  CUtensorMap tw;
  std::memset(&tw, 0, sizeof tw);
  if (kWT && !make_tmap(&tw, p.w_t, WKV_F32, p.B, p.T, p.C, L, kChunkCG)) return WKV_ERR_CUDA;
  const size_t smem = 2ull * L * kChunkCG * sizeof(KV) + (kWT ? sizeof(float) * L * kChunkCG : 0) +
                      sizeof(float4) * NW * kChunkCG + (kWT ? sizeof(float) * NW * kChunkCG : 0) + 64;
  auto fa = wkv_tile_totals<KV, NW, J, kWT>;
  int occ = 0;
  if (!kernel_setup(fa, dev, NW * 32, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  const long long BNG = (long long)p.B * p.NG;
  if (p.nch > 1) {
    fa<<<(unsigned)((p.nch - 1) * BNG), NW * 32, smem, st>>>(p, tk, tv, tw);
    if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  }
  // segments per channel in the scan: at most about 16 chunk totals each
  const int ntot = p.nch - 1;
  int seg = pl.scan_segments;
  if (seg == 0) seg = ntot <= 16 ? 1 : (ntot <= 64 ? 4 : (ntot <= 256 ? 16 : 64));
  const unsigned gs = (unsigned)(BNG * 4);  // 16 channels per CTA
  // programmatic serialization only behind A (an ordinary launch, so S is
  // scheduled only after the launch ahead of the call has ended: S reads w
  // before its own wait)
  PdlConfig cs(dim3(gs), dim3(16 * seg), 0, st);
  if (p.nch <= 1) cs.cfg.numAttrs = 0;
  cudaError_t e;
  switch (seg) {
    case 1: e = cudaLaunchKernelEx(&cs.cfg, wkv_tile_scan<1, kWT>, p, L); break;
    case 4: e = cudaLaunchKernelEx(&cs.cfg, wkv_tile_scan<4, kWT>, p, L); break;
    case 16: e = cudaLaunchKernelEx(&cs.cfg, wkv_tile_scan<16, kWT>, p, L); break;
    default: e = cudaLaunchKernelEx(&cs.cfg, wkv_tile_scan<64, kWT>, p, L); break;
  }
  if (!cuda_ok(e) || launch_result() != WKV_OK) return WKV_ERR_CUDA;
  // B: the sequential kernel over every (batch row, chunk, 32-channel group),
  // from the chunk's incoming state; one channel per thread
  constexpr bool kF32 = sizeof(KV) == 4;
  constexpr int LT = kF32 ? 2 * kSeqLtF32 : 2 * kSeqLtBf16;
  // one channel per thread, replay_threads channels per CTA (32 with
  // per-token decays)
  const int th = kWT ? 32 : pl.replay_threads;
  CUtensorMap bk, bv, bw;
  if (!make_tmap(&bk, p.k, kvdt, p.B, p.T, p.C, LT, th) || !make_tmap(&bv, p.v, kvdt, p.B, p.T, p.C, LT, th))
    return WKV_ERR_CUDA;
  // a replay of at most two stages is prefetched whole with 2 (more CTAs fit
  // per SM); longer ones stream through 3
  FwdParams q = p;
  q.replay_chunks = pl.replay_chunks;
  const bool two = pl.replay_chunks * L <= 2 * LT;
  if (kWT) {
    if (!make_tmap(&bw, p.w_t, WKV_F32, p.B, p.T, p.C, LT, th)) return WKV_ERR_CUDA;
    return two ? launch_seq_chunks<KV, OUT, 32, LT, 2, true>(q, bk, bv, st, dev, &bw)
               : launch_seq_chunks<KV, OUT, 32, LT, 3, true>(q, bk, bv, st, dev, &bw);
  } else {
    if (kF32 && pl.replay_chunks * L == 32 && th == 32) {
      // a 32-token fp32 replay as one 32-token stage: one copy pair and one
      // wait instead of two (layer: 23.5 against 23.8 us)
      CUtensorMap ck, cv;
      if (!make_tmap(&ck, p.k, kvdt, p.B, p.T, p.C, 32, th) || !make_tmap(&cv, p.v, kvdt, p.B, p.T, p.C, 32, th))
        return WKV_ERR_CUDA;
      return launch_seq_chunks<KV, OUT, 32, 32, 1>(q, ck, cv, st, dev);
    }
    switch (th) {
      case 64:
        return two ? launch_seq_chunks<KV, OUT, 64, LT, 2>(q, bk, bv, st, dev)
                   : launch_seq_chunks<KV, OUT, 64, LT, 3>(q, bk, bv, st, dev);
      case 128:
        return two ? launch_seq_chunks<KV, OUT, 128, LT, 2>(q, bk, bv, st, dev)
                   : launch_seq_chunks<KV, OUT, 128, LT, 3>(q, bk, bv, st, dev);
      default:
        return two ? launch_seq_chunks<KV, OUT, 32, LT, 2>(q, bk, bv, st, dev)
                   : launch_seq_chunks<KV, OUT, 32, LT, 3>(q, bk, bv, st, dev);
    }
  }
}

template <typename KV, typename OUT>
wkv_status launch_tile3_shape(const Plan& pl, const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                              wkv_dtype kvdt, cudaStream_t st, int dev) {
  if (p.w_t) {  // make_plan takes 16-token spans with per-token decays
    switch (pl.L) {
      case 32: return launch_tile3<KV, OUT, 2, 16, true>(pl, p, tk, tv, kvdt, st, dev);
      case 64: return launch_tile3<KV, OUT, 4, 16, true>(pl, p, tk, tv, kvdt, st, dev);
      default: return launch_tile3<KV, OUT, 8, 16, true>(pl, p, tk, tv, kvdt, st, dev);
    }
  }
  if (pl.J == 8) {
    switch (pl.L) {
      case 32: return launch_tile3<KV, OUT, 4, 8, false>(pl, p, tk, tv, kvdt, st, dev);
      case 64: return launch_tile3<KV, OUT, 8, 8, false>(pl, p, tk, tv, kvdt, st, dev);
      default: return launch_tile3<KV, OUT, 16, 8, false>(pl, p, tk, tv, kvdt, st, dev);
    }
  }
  switch (pl.L) {
    case 32: return launch_tile3<KV, OUT, 2, 16, false>(pl, p, tk, tv, kvdt, st, dev);
    case 64: return launch_tile3<KV, OUT, 4, 16, false>(pl, p, tk, tv, kvdt, st, dev);
    default: return launch_tile3<KV, OUT, 8, 16, false>(pl, p, tk, tv, kvdt, st, dev);
  }
}

template <typename KV, typename OUT, bool kTMA>
wkv_status launch_chunk_shape(const Plan& pl, const FwdParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                              cudaStream_t st, int dev) {
  if (pl.J == 8) {
    switch (pl.L) {
      case 32: return launch_chunk<KV, OUT, 4, 8, kTMA>(p, tk, tv, st, dev);
      case 64: return launch_chunk<KV, OUT, 8, 8, kTMA>(p, tk, tv, st, dev);
      default: return launch_chunk<KV, OUT, 16, 8, kTMA>(p, tk, tv, st, dev);
    }
  }
  switch (pl.L) {
    case 32: return launch_chunk<KV, OUT, 2, 16, kTMA>(p, tk, tv, st, dev);
    case 64: return launch_chunk<KV, OUT, 4, 16, kTMA>(p, tk, tv, st, dev);
    default: return launch_chunk<KV, OUT, 8, 16, kTMA>(p, tk, tv, st, dev);
  }
}

// The sequential kernel with TMA-fed stages of VEC channels per thread. A
// stage holds about 4 KB of k and v whatever VEC is (fewer channels, more
// tokens).
template <typename KV, typename OUT, int VEC>
wkv_status launch_seq_tma(const Plan& pl, const FwdParams& p, wkv_dtype kvdt, cudaStream_t st, int dev) {
  constexpr bool kF32 = sizeof(KV) == 4;
  constexpr int LT = (kF32 ? kSeqLtF32 : kSeqLtBf16) * (2 / VEC);
  // one channel per thread: 3 stages (12 KB), so that the many one-warp CTAs
  // this variant is for all fit on the device at once
  constexpr int STG = VEC == 1 ? 3 : (kF32 ? kSeqStagesF32 : kSeqStagesBf16);
  CUtensorMap tk, tv;
  const int cg = pl.seq_threads * VEC;
  if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, LT, cg) || !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, LT, cg))
    return WKV_ERR_CUDA;
  switch (pl.seq_threads) {
    case 32: return launch_seq<KV, OUT, 32, VEC, LT, STG, true>(p, tk, tv, tv, st, dev);
    case 64: return launch_seq<KV, OUT, 64, VEC, LT, STG, true>(p, tk, tv, tv, st, dev);
    default: return launch_seq<KV, OUT, 128, VEC, LT, STG, true>(p, tk, tv, tv, st, dev);
  }
}

// The sequential kernel with per-token decays: one channel per thread,
// 32-thread CTAs, k, v and w_t in TMA-fed stages of 16 (fp32) or 32 (bf16)
// tokens, 3 stages.
template <typename KV, typename OUT>
wkv_status launch_seq_tma_wt(const FwdParams& p, wkv_dtype kvdt, cudaStream_t st, int dev) {
  constexpr bool kF32 = sizeof(KV) == 4;
  constexpr int LT = kF32 ? 2 * kSeqLtF32 : 2 * kSeqLtBf16;
  CUtensorMap tk, tv, tw;
  if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, LT, 32) || !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, LT, 32) ||
      !make_tmap(&tw, p.w_t, WKV_F32, p.B, p.T, p.C, LT, 32))
    return WKV_ERR_CUDA;
  return launch_seq<KV, OUT, 32, 1, LT, 3, true, true>(p, tk, tv, tw, st, dev);
}

// The cluster scan: clusters of pl.ncl CTAs, one per (segment, batch row,
// 32-channel group); each warp's ring is fed by TMA boxes of kClusterLB
// tokens x 32 channels.
template <typename KV, typename OUT, int NW, int J, bool kWT>
wkv_status launch_cluster(const Plan& pl, const FwdParams& p, cudaStream_t st, int dev, wkv_dtype kvdt) {
  constexpr size_t smem = cluster_smem_bytes<KV, NW, kWT>();
  auto fn = wkv_fwd_cluster<KV, OUT, NW, J, kWT>;
  int occ = 0;
  if (!kernel_setup(fn, dev, NW * 32, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  CUtensorMap tk, tv, tw;
  if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, kClusterLB, 32) ||
      !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, kClusterLB, 32))
    return WKV_ERR_CUDA;
  if (kWT) {
    if (!make_tmap(&tw, p.w_t, WKV_F32, p.B, p.T, p.C, kClusterLB, 32)) return WKV_ERR_CUDA;
  } else {
    tw = tk;  // unused
  }
  FwdParams q = p;
  q.cluster = pl.ncl;
  q.nseg = pl.nseg;
  const long long items = (long long)p.B * ((p.C + 31) / 32);
  const long long grid = items * pl.nseg * pl.ncl;
  if (grid >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)pl.ncl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!cuda_ok(cudaLaunchKernelEx(&cfg, fn, q, tk, tv, tw))) return WKV_ERR_CUDA;
  return launch_result();
}

template <typename KV, typename OUT, bool kWT>
wkv_status launch_cluster_shape(const Plan& pl, const FwdParams& p, cudaStream_t st, int dev, wkv_dtype kvdt) {
  if (pl.cj == 32) {
    return pl.cw == 4 ? launch_cluster<KV, OUT, 4, 32, kWT>(pl, p, st, dev, kvdt)
                      : launch_cluster<KV, OUT, 8, 32, kWT>(pl, p, st, dev, kvdt);
  }
  return pl.cw == 4 ? launch_cluster<KV, OUT, 4, 64, kWT>(pl, p, st, dev, kvdt)
                    : launch_cluster<KV, OUT, 8, 64, kWT>(pl, p, st, dev, kvdt);
}

template <typename KV, typename OUT>
wkv_status dispatch_forward(const Plan& pl, FwdParams& p, bool tma, wkv_dtype kvdt, cudaStream_t st, int dev,
                            const DevInfo& di) {
  CUtensorMap tk, tv;
  std::memset(&tk, 0, sizeof tk);
  std::memset(&tv, 0, sizeof tv);
  if (pl.kernel == 5) {
    return p.w_t ? launch_cluster_shape<KV, OUT, true>(pl, p, st, dev, kvdt)
                 : launch_cluster_shape<KV, OUT, false>(pl, p, st, dev, kvdt);
  }
  if (pl.kernel == 1) {
    if (p.w_t) {
      // per-token decays: one channel per thread, 32-thread CTAs
      if (tma) return launch_seq_tma_wt<KV, OUT>(p, kvdt, st, dev);
      return launch_seq<KV, OUT, 128, kSeqFallbackVec, kSeqFallbackLt, 1, false, true>(p, tk, tv, tv, st, dev);
    }
    if (tma) {
      if (pl.seq_vec == 1) return launch_seq_tma<KV, OUT, 1>(pl, p, kvdt, st, dev);
      return launch_seq_tma<KV, OUT, 2>(pl, p, kvdt, st, dev);
    }
    return launch_seq<KV, OUT, 128, kSeqFallbackVec, kSeqFallbackLt, 1, false, false>(p, tk, tv, tv, st, dev);
  }
  if (pl.kernel == 3) {  // three launches (make_plan only chooses it when TMA works)
    if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, pl.L, kChunkCG) ||
        !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, pl.L, kChunkCG))
      return WKV_ERR_CUDA;
    return launch_tile3_shape<KV, OUT>(pl, p, tk, tv, kvdt, st, dev);
  }
  if (pl.kernel == 4) {  // pipelined (make_plan only chooses it when TMA works)
    if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, pl.L, kChunkCG) ||
        !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, pl.L, kChunkCG))
      return WKV_ERR_CUDA;
    return launch_pipe_shape<KV, OUT>(pl, p, tk, tv, st, dev, di);
  }
  if (tma) {
    if (!make_tmap(&tk, p.k, kvdt, p.B, p.T, p.C, pl.L, kChunkCG) ||
        !make_tmap(&tv, p.v, kvdt, p.B, p.T, p.C, pl.L, kChunkCG))
      return WKV_ERR_CUDA;
    return launch_chunk_shape<KV, OUT, true>(pl, p, tk, tv, st, dev);
  }
  return launch_chunk_shape<KV, OUT, false>(pl, p, tk, tv, st, dev);
}

// ---------------------------------------------------------------------------
// RWKV-v6 matrix-valued state
// ---------------------------------------------------------------------------
// [rows, cols] row-major tensor, box [box_rows, box_cols]
bool make_tmap_2d(CUtensorMap* m, const void* base, wkv_dtype dt, int64_t rows, int64_t cols, int box_rows,
                  int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const size_t es = dt == WKV_F32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * es)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt == WKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kV6Tokens = 32;  // tokens per staged block

template <typename KV, typename OUT, int D>
wkv_status launch_v6(const V6Params& p, const void* r, const float* w, const void* k, const void* v, wkv_dtype kvdt,
                     cudaStream_t st, int dev) {
  constexpr int RB = V6Shape<KV, D>::kRows;  // state rows per CTA
  const int64_t rows = (int64_t)p.B * p.T, cols = (int64_t)p.H * D;
  CUtensorMap tk, tv, tr, tw;
  if (!make_tmap_2d(&tk, k, kvdt, rows, cols, kV6Tokens, D) || !make_tmap_2d(&tv, v, kvdt, rows, cols, kV6Tokens, D) ||
      !make_tmap_2d(&tr, r, kvdt, rows, cols, kV6Tokens, RB) ||
      !make_tmap_2d(&tw, w, WKV_F32, rows, cols, kV6Tokens, RB))
    return WKV_ERR_CUDA;
  const size_t smem = 2 * v6_stage_bytes<KV, D, RB, kV6Tokens>() + 16;
  auto fn = wkv6_fwd<KV, OUT, D, RB>;
  int occ = 0;
  if (!kernel_setup(fn, dev, 128, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
  const long long grid = (long long)p.B * p.H * (D / RB);
  if (grid >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  fn<<<(unsigned)grid, 128, smem, st>>>(p, tk, tv, tr, tw);
  return launch_result();
}

template <typename KV, typename OUT>
wkv_status launch_v6_d(int64_t D, const V6Params& p, const void* r, const float* w, const void* k, const void* v,
                       wkv_dtype kvdt, cudaStream_t st, int dev) {
  switch (D) {
    case 32: return launch_v6<KV, OUT, 32>(p, r, w, k, v, kvdt, st, dev);
    case 64: return launch_v6<KV, OUT, 64>(p, r, w, k, v, kvdt, st, dev);
    default: return launch_v6<KV, OUT, 128>(p, r, w, k, v, kvdt, st, dev);
  }
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------
// tokens per chunk of the backward (measured: 16 against 32 tokens, layer
// 95.8 against 103.2 us, long 1.68 against 1.87 ms; the gradient pass's
// one-warp CTAs hold half the shared memory, so twice as many fit per SM)
constexpr int kBwdL = 16;

struct BwdPlan {
  int NG, nch;
  size_t off_agg, off_x0, off_rtot, off_rin, off_pdu, off_pdw, bytes;
};

bool make_bwd_plan(int64_t B, int64_t T, int64_t C, BwdPlan* pl) {
  std::memset(pl, 0, sizeof *pl);
  if (!sizes_ok(B, T, C)) return false;
  pl->NG = (int)((C + kChunkCG - 1) / kChunkCG);
  pl->nch = (int)std::max<int64_t>(1, (T + kBwdL - 1) / kBwdL);
  const size_t slots = (size_t)B * pl->NG * kChunkCG;  // float4 slots per chunk
  size_t off = sizeof(WsHeader);
  pl->off_agg = off;
  off = round_up(off + sizeof(float4) * slots * (size_t)std::max(pl->nch - 1, 1), 256);
  pl->off_x0 = off;
  off = round_up(off + sizeof(float4) * slots * pl->nch, 256);
  pl->off_rtot = off;
  off = round_up(off + sizeof(float4) * slots * pl->nch, 256);
  pl->off_rin = off;
  off = round_up(off + sizeof(float4) * slots * pl->nch, 256);
  pl->off_pdu = off;
  off = round_up(off + sizeof(float) * (size_t)pl->nch * B * C, 256);
  pl->off_pdw = off;
  off = round_up(off + sizeof(float) * (size_t)pl->nch * B * C, 256);
  pl->bytes = off;
  return true;
}

template <int SEG_MAX>
int scan_segments_for(int ntot) {
  const int seg = ntot <= 16 ? 1 : (ntot <= 64 ? 4 : (ntot <= 256 ? 16 : 64));
  return std::min(seg, SEG_MAX);
}

template <typename KV>
wkv_status launch_backward(const BwdPlan& pl, const FwdParams& fp, const BwdParams& bp, wkv_dtype kvdt,
                           cudaStream_t st, int dev) {
  // A, S: the forward state entering every chunk (the forward's passes)
  constexpr int NW = kBwdL / 16, J = 16;
  const long long BNG = (long long)fp.B * fp.NG;
  if (pl.nch > 1) {
    CUtensorMap tk, tv;
    if (!make_tmap(&tk, fp.k, kvdt, fp.B, fp.T, fp.C, kBwdL, kChunkCG) ||
        !make_tmap(&tv, fp.v, kvdt, fp.B, fp.T, fp.C, kBwdL, kChunkCG))
      return WKV_ERR_CUDA;
    const size_t smem = 2ull * kBwdL * kChunkCG * sizeof(KV) + sizeof(float4) * NW * kChunkCG + 64;
    auto fa = wkv_tile_totals<KV, NW, J, false>;
    int occ = 0;
    if (!kernel_setup(fa, dev, NW * 32, smem, &occ) || occ < 1) return WKV_ERR_CUDA;
    fa<<<(unsigned)((pl.nch - 1) * BNG), NW * 32, smem, st>>>(fp, tk, tv, tv);
    if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  }
  const int seg = scan_segments_for<64>(pl.nch - 1);
  const unsigned gs = (unsigned)(BNG * 4);
  switch (seg) {
    case 1: wkv_tile_scan<1, false><<<gs, 16, 0, st>>>(fp, kBwdL); break;
    case 4: wkv_tile_scan<4, false><<<gs, 64, 0, st>>>(fp, kBwdL); break;
    case 16: wkv_tile_scan<16, false><<<gs, 256, 0, st>>>(fp, kBwdL); break;
    default: wkv_tile_scan<64, false><<<gs, 1024, 0, st>>>(fp, kBwdL); break;
  }
  if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  // the chunks' k, v, g tiles (32 channels x kBwdL tokens) for R1 and R2
  CUtensorMap rk, rv, rg;
  if (!make_tmap(&rk, fp.k, kvdt, fp.B, fp.T, fp.C, kBwdL, 32) ||
      !make_tmap(&rv, fp.v, kvdt, fp.B, fp.T, fp.C, kBwdL, 32) ||
      !make_tmap(&rg, bp.g, WKV_F32, fp.B, fp.T, fp.C, kBwdL, 32))
    return WKV_ERR_CUDA;
  const size_t tsmem = bwd_tile_bytes<KV, kBwdL>() + 16;
  // R1: reverse aggregates of chunks 1 .. nch-1
  const long long ngw = (fp.C + 31) / 32;
  if (pl.nch > 1) {
    const long long items = (long long)fp.B * (pl.nch - 1) * ngw;
    if (items >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
    wkv_bwd_rev_totals<KV, kBwdL><<<(unsigned)items, 32, tsmem, st>>>(bp, rk, rv, rg);
    if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  }
  // RS: the reverse state entering every chunk from its end
  switch (seg) {
    case 1: wkv_bwd_rev_scan<1><<<gs, 16, 0, st>>>(bp); break;
    case 4: wkv_bwd_rev_scan<4><<<gs, 64, 0, st>>>(bp); break;
    case 16: wkv_bwd_rev_scan<16><<<gs, 256, 0, st>>>(bp); break;
    default: wkv_bwd_rev_scan<64><<<gs, 1024, 0, st>>>(bp); break;
  }
  if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  // R2: the gradients
  const long long items = (long long)fp.B * pl.nch * ngw;
  if (items >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  wkv_bwd_chunk<KV, kBwdL><<<(unsigned)items, 32, tsmem, st>>>(bp, rk, rv, rg);
  if (launch_result() != WKV_OK) return WKV_ERR_CUDA;
  // RED: du, dw (one warp per channel)
  wkv_bwd_reduce<<<(unsigned)((fp.C + 7) / 8), 256, 0, st>>>(bp);
  return launch_result();
}

}  // namespace
}  // namespace wkv

using namespace wkv;

extern "C" {

int32_t wkv_version(void) { return 100; }

const char* wkv_last_cuda_error(void) { return cudaGetErrorName(g_last_cuda_error); }

const char* wkv_status_string(wkv_status s) {
  switch (s) {
    case WKV_OK: return "ok";
    case WKV_ERR_INVALID_ARG: return "invalid argument";
    case WKV_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype combination";
    case WKV_ERR_MISALIGNED: return "misaligned pointer";
    case WKV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case WKV_ERR_CUDA: return "CUDA runtime error";
    case WKV_ERR_WAIT_TIMEOUT: return "device-side wait timed out";
    case WKV_ERR_BOUNDS: return "device-side index out of bounds (bounds-checked build)";
  }
  return "unknown status";
}

size_t wkv_forward_workspace_size(int64_t B, int64_t T, int64_t C, const wkv_options* opts) {
  // the automatic choice of kernel may depend on the input dtype, which is
  // not an argument here: return what either choice needs
  Plan pl;
  if (!sizes_ok(B, T, C) || !make_plan(B, T, C, opts, &pl)) return 0;
  return pl.bytes;
}

int32_t wkv_forward_kernel(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, const wkv_options* opts) {
  if (!sizes_ok(B, T, C)) return 0;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return 0;
  const size_t es = kv_dtype == WKV_F32 ? 4 : 2;
  Plan pl;
  if (!make_plan(B, T, C, opts, &pl, (C * (int64_t)es) % 16 == 0)) return 0;
  return pl.kernel;
}

int32_t wkv_forward_launches(int64_t B, int64_t T, int64_t C, wkv_dtype kv_dtype, const wkv_options* opts) {
  if (!sizes_ok(B, T, C) || B * C == 0 || T == 0) return 0;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return 0;
  const size_t es = kv_dtype == WKV_F32 ? 4 : 2;
  Plan pl;
  if (!make_plan(B, T, C, opts, &pl, (C * (int64_t)es) % 16 == 0)) return 0;
  if (pl.kernel == 3) return pl.nch > 1 ? 3 : 2;  // chunk totals (when there is more than one chunk), scan, replay
  return 1;
}

wkv_status wkv_forward_ext(int64_t B, int64_t T, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype,
                           const float* w, const float* u, void* out, wkv_dtype out_dtype,
                           const wkv_cstate* state_in, const wkv_state* state_out, void* workspace,
                           size_t workspace_bytes, void* stream, const wkv_options* opts, const wkv_ext* ext) {
  const float* w_t = ext ? ext->w_t : nullptr;
  const void* r = ext ? ext->r : nullptr;
  // ---- argument checks: nothing is launched before they pass
  const wkv_status chk =
      check_forward_args(B, T, C, k, v, kv_dtype, w_t ? u : w, u, out, out_dtype, state_in, state_out, opts);
  if (chk != WKV_OK) return chk;
  if (B * T * C > 0 && (w_t || r) && !aligned(w_t ? (const void*)w_t : r, 4)) return WKV_ERR_INVALID_ARG;
  const size_t kes = kv_dtype == WKV_F32 ? 4 : 2;
  // TMA needs 16-byte aligned bases and row pitches; otherwise the kernels
  // fill their tiles with plain loads
  const bool tma = tma_usable(k, v, C, kes) && (!w_t || tma_usable(w_t, w_t, C, 4));
  Plan pl;
  if (!make_plan(B, T, C, opts, &pl, tma, w_t != nullptr)) return WKV_ERR_INVALID_ARG;
  if (!workspace) return WKV_ERR_INVALID_ARG;
  if (workspace_bytes < pl.bytes) return WKV_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(workspace, 256)) return WKV_ERR_MISALIGNED;

  const int64_t BC = B * C;
  if (BC == 0) return WKV_OK;  // nothing to compute or write

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev))) return WKV_ERR_CUDA;
  DevInfo di;
  if (!dev_info(dev, &di)) return WKV_ERR_CUDA;
  if (T == 0) {  // the state passes through unchanged
    if (!state_out) return WKV_OK;
    if (state_in) {
      const float* src[3] = {state_in->num, state_in->den, state_in->max_e};
      float* dst[3] = {state_out->num, state_out->den, state_out->max_e};
      for (int i = 0; i < 3; ++i)
        if (src[i] != dst[i] &&
            !cuda_ok(cudaMemcpyAsync(dst[i], src[i], sizeof(float) * BC, cudaMemcpyDeviceToDevice, st)))
          return WKV_ERR_CUDA;
      return WKV_OK;
    }
    wkv_fill_empty_state<<<(unsigned)((BC + 255) / 256), 256, 0, st>>>(BC, state_out->num, state_out->den,
                                                                      state_out->max_e);
    return launch_result();
  }

  FwdParams p;
  std::memset(&p, 0, sizeof p);
  p.B = (int)B;
  p.T = (int)T;
  p.C = (int)C;
  p.k = k;
  p.v = v;
  p.w = w;
  p.u = u;
  p.out = out;
  p.w_t = w_t;
  p.r = r;
  if (state_in) {
    p.s_num = state_in->num;
    p.s_den = state_in->den;
    p.s_max = state_in->max_e;
  }
  if (state_out) {
    p.o_num = state_out->num;
    p.o_den = state_out->den;
    p.o_max = state_out->max_e;
  }
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.hdr = reinterpret_cast<WsHeader*>(ws);
  p.timeout_ns = (opts && opts->wait_timeout_ns > 0) ? (uint64_t)opts->wait_timeout_ns : kDefaultTimeoutNs;
  p.inject_tile = (opts && opts->inject_enable) ? (int)std::min<int64_t>(opts->inject_unpublished_tile, INT32_MAX) : -1;
  if (pl.kernel == 5) {
    p.flags_a = reinterpret_cast<uint32_t*>(ws + pl.off_flags_a);
    p.agg_a = reinterpret_cast<float4*>(ws + pl.off_agg_a);
  } else if (pl.kernel >= 2) {
    p.NG = pl.NG;
    p.nch = pl.nch;
    p.G = pl.G;
    p.chunk_len = pl.L;
    p.n_tiles = (int)pl.n_tiles;
    p.flags_a = reinterpret_cast<uint32_t*>(ws + pl.off_flags_a);
    p.flags_p = reinterpret_cast<uint32_t*>(ws + pl.off_flags_p);
    p.agg_a = reinterpret_cast<float4*>(ws + pl.off_agg_a);
    p.agg_p = reinterpret_cast<float4*>(ws + pl.off_agg_p);
    if (pl.kernel == 3) {
      p.flags_a = p.flags_p = nullptr;
      p.x0 = reinterpret_cast<float4*>(ws + pl.off_x0);
      p.wtot = reinterpret_cast<float*>(ws + pl.off_wtot);
    }
  }
  const size_t oes = out_dtype == WKV_F32 ? 4 : 2;
  const int vec = pl.kernel == 1 ? (tma ? pl.seq_vec : kSeqFallbackVec)
                                 : kChunkVec;
  p.vec_store = aligned(out, oes * vec) && (C % vec) == 0;
  if (pl.kernel >= 2)  // the chunked kernels also load k and v VEC-wide
    p.vec_store = p.vec_store && aligned(k, kes * vec) && aligned(v, kes * vec);

  if (kv_dtype == WKV_F32) return dispatch_forward<float, float>(pl, p, tma, kv_dtype, st, dev, di);
  if (out_dtype == WKV_BF16)
    return dispatch_forward<__nv_bfloat16, __nv_bfloat16>(pl, p, tma, kv_dtype, st, dev, di);
  return dispatch_forward<__nv_bfloat16, float>(pl, p, tma, kv_dtype, st, dev, di);
}

wkv_status wkv_forward(int64_t B, int64_t T, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype,
                       const float* w, const float* u, void* out, wkv_dtype out_dtype, const wkv_cstate* state_in,
                       const wkv_state* state_out, void* workspace, size_t workspace_bytes, void* stream,
                       const wkv_options* opts) {
  return wkv_forward_ext(B, T, C, k, v, kv_dtype, w, u, out, out_dtype, state_in, state_out, workspace,
                         workspace_bytes, stream, opts, nullptr);
}

wkv_status wkv_step_ext(int64_t S, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype, const float* w,
                        const float* u, void* out, wkv_dtype out_dtype, const wkv_cstate* state_in,
                        const wkv_state* state_out, void* stream, const wkv_ext* ext) {
  const float* w_t = ext ? ext->w_t : nullptr;
  const void* r = ext ? ext->r : nullptr;
  if (S < 0 || C < 0) return WKV_ERR_INVALID_ARG;
  if (S > 0 && C > (int64_t)((1ull << 62) / (uint64_t)S)) return WKV_ERR_INVALID_ARG;
  if (C >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (out_dtype != WKV_F32 && out_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (kv_dtype == WKV_F32 && out_dtype != WKV_F32) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (!state_in || !state_out) return WKV_ERR_INVALID_ARG;
  if (!state_in->num || !state_in->den || !state_in->max_e) return WKV_ERR_INVALID_ARG;
  if (!state_out->num || !state_out->den || !state_out->max_e) return WKV_ERR_INVALID_ARG;
  const int64_t n = S * C;
  if (n == 0) return WKV_OK;
  if (!k || !v || (!w && !w_t) || !u || !out) return WKV_ERR_INVALID_ARG;

  StepParams p;
  p.n = n;
  p.C = (int)C;
  p.k = k;
  p.v = v;
  p.w = w;
  p.u = u;
  p.out = out;
  p.s_num = state_in->num;
  p.s_den = state_in->den;
  p.s_max = state_in->max_e;
  p.o_num = state_out->num;
  p.o_den = state_out->den;
  p.o_max = state_out->max_e;
  p.w_t = w_t;
  p.r = r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t kes = kv_dtype == WKV_F32 ? 4 : 2, oes = out_dtype == WKV_F32 ? 4 : 2;
  constexpr int VEC = 4;
  const bool vec = (C % VEC) == 0 && aligned(k, kes * VEC) && aligned(v, kes * VEC) && aligned(out, oes * VEC) &&
                   (w_t ? aligned(w_t, 16) : aligned(w, 16)) && (!r || aligned(r, kes * VEC)) && aligned(u, 16) &&
                   aligned(p.s_num, 16) && aligned(p.s_den, 16) && aligned(p.s_max, 16) && aligned(p.o_num, 16) &&
                   aligned(p.o_den, 16) && aligned(p.o_max, 16);
  const int per = vec ? VEC : 1;
  const long long threads = (n + per - 1) / per;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (kv_dtype == WKV_F32) {
    if (vec) wkv_step_kernel<float, float, VEC><<<blocks, 256, 0, st>>>(p);
    else wkv_step_kernel<float, float, 1><<<blocks, 256, 0, st>>>(p);
  } else if (out_dtype == WKV_BF16) {
    if (vec) wkv_step_kernel<__nv_bfloat16, __nv_bfloat16, VEC><<<blocks, 256, 0, st>>>(p);
    else wkv_step_kernel<__nv_bfloat16, __nv_bfloat16, 1><<<blocks, 256, 0, st>>>(p);
  } else {
    if (vec) wkv_step_kernel<__nv_bfloat16, float, VEC><<<blocks, 256, 0, st>>>(p);
    else wkv_step_kernel<__nv_bfloat16, float, 1><<<blocks, 256, 0, st>>>(p);
  }
  return launch_result();
}

wkv_status wkv_step(int64_t S, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype, const float* w,
                    const float* u, void* out, wkv_dtype out_dtype, const wkv_cstate* state_in,
                    const wkv_state* state_out, void* stream) {
  return wkv_step_ext(S, C, k, v, kv_dtype, w, u, out, out_dtype, state_in, state_out, stream, nullptr);
}

wkv_status wkv_v6_forward(int64_t B, int64_t T, int64_t H, int64_t D, const void* r, const float* w, const void* k,
                        const void* v, wkv_dtype kv_dtype, void* y, wkv_dtype y_dtype, const float* state_in,
                        float* state_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || T < 0 || H < 0) return WKV_ERR_INVALID_ARG;
  if (D != 32 && D != 64 && D != 128) return WKV_ERR_INVALID_ARG;
  if (T >= (1ll << 24) || H >= (1ll << 20) || B >= (1ll << 31)) return WKV_ERR_INVALID_ARG;
  if (B > 0 && H > 0 && T > (int64_t)((1ull << 40) / (uint64_t)(B * H))) return WKV_ERR_INVALID_ARG;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (y_dtype != WKV_F32 && y_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (kv_dtype == WKV_F32 && y_dtype != WKV_F32) return WKV_ERR_UNSUPPORTED_DTYPE;
  const int64_t n = B * T * H * D;
  if (n > 0 && (!r || !w || !k || !v || !y)) return WKV_ERR_INVALID_ARG;
  if (!workspace) return WKV_ERR_INVALID_ARG;
  if (workspace_bytes < sizeof(WsHeader)) return WKV_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(workspace, 256)) return WKV_ERR_MISALIGNED;
  // TMA: 16-byte aligned bases (the row pitch H*D*size is a multiple of 16 for D >= 32)
  if (n > 0 && (!aligned(r, 16) || !aligned(w, 16) || !aligned(k, 16) || !aligned(v, 16))) return WKV_ERR_MISALIGNED;
  if (B * H == 0) return WKV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // the state passes through
    if (state_out && state_out != state_in) {
      const size_t bytes = sizeof(float) * (size_t)(B * H * D * D);
      if (state_in) {
        if (!cuda_ok(cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, st))) return WKV_ERR_CUDA;
      } else if (!cuda_ok(cudaMemsetAsync(state_out, 0, bytes, st))) {
        return WKV_ERR_CUDA;
      }
    }
    return WKV_OK;
  }
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev))) return WKV_ERR_CUDA;
  V6Params p;
  std::memset(&p, 0, sizeof p);
  p.B = (int)B;
  p.T = (int)T;
  p.H = (int)H;
  p.y = y;
  p.s_in = state_in;
  p.s_out = state_out;
  p.hdr = static_cast<WsHeader*>(workspace);
  p.timeout_ns = kDefaultTimeoutNs;
  if (kv_dtype == WKV_F32) return launch_v6_d<float, float>(D, p, r, w, k, v, kv_dtype, st, dev);
  if (y_dtype == WKV_BF16) return launch_v6_d<__nv_bfloat16, __nv_bfloat16>(D, p, r, w, k, v, kv_dtype, st, dev);
  return launch_v6_d<__nv_bfloat16, float>(D, p, r, w, k, v, kv_dtype, st, dev);
}

size_t wkv_backward_workspace_size(int64_t B, int64_t T, int64_t C) {
  BwdPlan pl;
  if (!make_bwd_plan(B, T, C, &pl)) return 0;
  return pl.bytes;
}

wkv_status wkv_backward(int64_t B, int64_t T, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype,
                        const float* w, const float* u, const wkv_cstate* state_in, const float* gout, float* dk,
                        float* dv, float* dw, float* du, const wkv_state* dstate_in, void* workspace,
                        size_t workspace_bytes, void* stream) {
  // ---- argument checks: nothing is launched before they pass
  if (!sizes_ok(B, T, C)) return WKV_ERR_INVALID_ARG;
  if (kv_dtype != WKV_F32 && kv_dtype != WKV_BF16) return WKV_ERR_UNSUPPORTED_DTYPE;
  if (state_in && (!state_in->num || !state_in->den || !state_in->max_e)) return WKV_ERR_INVALID_ARG;
  if (dstate_in && (!dstate_in->num || !dstate_in->den || !dstate_in->max_e)) return WKV_ERR_INVALID_ARG;
  if (B * T * C > 0 && (!k || !v || !gout || !dk || !dv)) return WKV_ERR_INVALID_ARG;
  if (C > 0 && (!w || !u || !dw || !du)) return WKV_ERR_INVALID_ARG;
  const size_t kes = kv_dtype == WKV_F32 ? 4 : 2;
  BwdPlan pl;
  if (!make_bwd_plan(B, T, C, &pl)) return WKV_ERR_INVALID_ARG;
  if (!workspace) return WKV_ERR_INVALID_ARG;
  if (workspace_bytes < pl.bytes) return WKV_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(workspace, 256)) return WKV_ERR_MISALIGNED;
  // the kernels copy k, v and gout with TMA
  if (B * T * C > 0 && (!tma_usable(k, v, C, kes) || !tma_usable(gout, gout, C, 4))) return WKV_ERR_MISALIGNED;
  if (C == 0) return WKV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || T == 0) {
    // no tokens: every gradient is zero
    if (!cuda_ok(cudaMemsetAsync(dw, 0, sizeof(float) * C, st)) ||
        !cuda_ok(cudaMemsetAsync(du, 0, sizeof(float) * C, st)))
      return WKV_ERR_CUDA;
    if (dstate_in && B > 0) {
      float* d[3] = {dstate_in->num, dstate_in->den, dstate_in->max_e};
      for (float* x : d)
        if (!cuda_ok(cudaMemsetAsync(x, 0, sizeof(float) * B * C, st))) return WKV_ERR_CUDA;
    }
    return WKV_OK;
  }
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev))) return WKV_ERR_CUDA;
  unsigned char* ws = static_cast<unsigned char*>(workspace);

  FwdParams fp;
  std::memset(&fp, 0, sizeof fp);
  fp.B = (int)B;
  fp.T = (int)T;
  fp.C = (int)C;
  fp.NG = pl.NG;
  fp.nch = pl.nch;
  fp.chunk_len = kBwdL;
  fp.k = k;
  fp.v = v;
  fp.w = w;
  fp.u = u;
  if (state_in) {
    fp.s_num = state_in->num;
    fp.s_den = state_in->den;
    fp.s_max = state_in->max_e;
  }
  fp.hdr = reinterpret_cast<WsHeader*>(ws);
  fp.timeout_ns = kDefaultTimeoutNs;
  fp.inject_tile = -1;
  fp.agg_a = reinterpret_cast<float4*>(ws + pl.off_agg);
  fp.x0 = reinterpret_cast<float4*>(ws + pl.off_x0);

  BwdParams bp;
  std::memset(&bp, 0, sizeof bp);
  bp.B = (int)B;
  bp.T = (int)T;
  bp.C = (int)C;
  bp.NG = pl.NG;
  bp.nch = pl.nch;
  bp.chunk_len = kBwdL;
  bp.k = k;
  bp.v = v;
  bp.w = w;
  bp.u = u;
  bp.g = gout;
  bp.s_num = fp.s_num;
  bp.s_den = fp.s_den;
  bp.s_max = fp.s_max;
  bp.dk = dk;
  bp.dv = dv;
  bp.dw = dw;
  bp.du = du;
  if (dstate_in) {
    bp.d_num = dstate_in->num;
    bp.d_den = dstate_in->den;
    bp.d_max = dstate_in->max_e;
  }
  bp.x0 = fp.x0;
  bp.rtot = reinterpret_cast<float4*>(ws + pl.off_rtot);
  bp.rin = reinterpret_cast<float4*>(ws + pl.off_rin);
  bp.pdu = reinterpret_cast<float*>(ws + pl.off_pdu);
  bp.pdw = reinterpret_cast<float*>(ws + pl.off_pdw);
  bp.hdr = fp.hdr;
  bp.timeout_ns = kDefaultTimeoutNs;
  if (kv_dtype == WKV_F32) return launch_backward<float>(pl, fp, bp, kv_dtype, st, dev);
  return launch_backward<__nv_bfloat16>(pl, fp, bp, kv_dtype, st, dev);
}

wkv_status wkv_query_status(void* workspace, void* stream) {
  if (!workspace) return WKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!cuda_ok(cudaStreamSynchronize(st))) return WKV_ERR_CUDA;
  WsHeader* h = static_cast<WsHeader*>(workspace);
  uint32_t bits = 0;
  if (!cuda_ok(cudaMemcpy(&bits, &h->status, sizeof bits, cudaMemcpyDeviceToHost))) return WKV_ERR_CUDA;
  if (bits) {
    const uint32_t zero = 0;
    if (!cuda_ok(cudaMemcpy(&h->status, &zero, sizeof zero, cudaMemcpyHostToDevice))) return WKV_ERR_CUDA;
  }
  if (bits & kStatusBoundsError) return WKV_ERR_BOUNDS;
  return (bits & kStatusWaitTimeout) ? WKV_ERR_WAIT_TIMEOUT : WKV_OK;
}

// ---------------------------------------------------------------------------
// wkv_forward_noalloc: wkv_forward with its scratch in a fixed device array
// ---------------------------------------------------------------------------
// For callers that cannot allocate device memory (a host that owns all of it
// and passes in only inputs and outputs; latency-bound code that must not take
// cudaMalloc's device-wide synchronisation). The array is zero at module load;
// each call zeroes the counters and flags its kernel relies on, then runs the
// ordinary forward path on the array. Calls share the array, so calls that
// overlap on the GPU race.
static __device__ __align__(256) unsigned char g_noalloc_scratch[WKV_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[wkv::kMaxDevices];

// Device address of g_noalloc_scratch on `dev` (the current device), looked up
// once per device. In host code the array's name is only a stand-in for the
// symbol, never a usable device address.
bool noalloc_scratch(int dev, void** ptr) {
  if (dev < 0 || dev >= wkv::kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(wkv::g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (!cuda_ok(cudaGetSymbolAddress(&p, g_noalloc_scratch)) || !p) return false;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return true;
}
}  // namespace

wkv_status wkv_forward_noalloc(int64_t B, int64_t T, int64_t C, const void* k, const void* v, wkv_dtype kv_dtype,
                               const float* w, const float* u, void* out, wkv_dtype out_dtype,
                               const wkv_cstate* state_in, const wkv_state* state_out, void* stream) {
  // every argument check of wkv_forward, before anything is queued on the stream
  const wkv_status chk =
      check_forward_args(B, T, C, k, v, kv_dtype, w, u, out, out_dtype, state_in, state_out, nullptr);
  if (chk != WKV_OK) return chk;
  Plan pl;
  const size_t kes = kv_dtype == WKV_BF16 ? 2 : 4;
  if (!make_plan(B, T, C, nullptr, &pl, tma_usable(k, v, C, kes))) return WKV_ERR_INVALID_ARG;
  if (pl.bytes > WKV_NOALLOC_SCRATCH_BYTES) return WKV_ERR_WORKSPACE_TOO_SMALL;
  if (B * C == 0) {
    // nothing to compute: wkv_forward checks the other arguments and returns
    // before it would look at a workspace, so no device (and no scratch
    // address) is needed; 256 only satisfies its alignment check
    return wkv_forward(B, T, C, k, v, kv_dtype, w, u, out, out_dtype, state_in, state_out,
                       reinterpret_cast<void*>(uintptr_t(256)), WKV_NOALLOC_SCRATCH_BYTES, stream, nullptr);
  }
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev))) return WKV_ERR_CUDA;
  void* scratch = nullptr;
  if (!noalloc_scratch(dev, &scratch)) return WKV_ERR_CUDA;
  // counters, epoch, status and flags start at zero for this call
  const size_t clear =
      (pl.kernel == 2 || pl.kernel == 4 || (pl.kernel == 5 && pl.nseg > 1)) ? pl.off_agg_a : sizeof(WsHeader);
  if (!cuda_ok(cudaMemsetAsync(scratch, 0, clear, reinterpret_cast<cudaStream_t>(stream))))
    return WKV_ERR_CUDA;
  return wkv_forward(B, T, C, k, v, kv_dtype, w, u, out, out_dtype, state_in, state_out, scratch,
                     WKV_NOALLOC_SCRATCH_BYTES, stream, nullptr);
}

}  // extern "C"
