// C-ABI host layer: argument checks, workspace carve-up, TMA descriptors, launches.
//
// One forward call: compaction of the valid rows -> vocabulary sweep (both block GEMMs,
// online LSE / KL epilogue, split-V partial state; with side outputs also the student
// entropy accumulator and the label logit) -> split-V merge -> [JSD: second sweep with the
// final LSEs -> partial-sum reduction] -> masked mean.
// One backward call: compaction -> per vocabulary chunk { gradient sweep writing the bf16
// gradient chunk G; grouped GEMM dh_s (+)= G W_s[chunk], dW_s[chunk] (+)= G^T h_s }.
// Vocabulary-parallel calls: the forward's sweep on one row shard of the unembeddings with
// the merged shard state as output, the cross-shard merge, and the JSD's second pass per shard.
// Spectral front end: Gram matrix and bf16 projections on the backward's GEMM kernel.
// Hand-off: a row copy from peer or IPC-mapped memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "nb_kl.h"
#include "common.cuh"
#include "gemm.cuh"
#include "rowops.cuh"
#include "sweep.cuh"

using namespace nbkl;

namespace {

constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per pipeline wait
constexpr int kTilesPerUnitFwd = 8;                          // 2048 vocabulary columns per unit
constexpr int kTilesPerUnitGrad = 4;                         // gradient sweep: 1024 columns per unit
constexpr int kTailItems = 160;   // single-tile work items at the end of a sweep (~2 waves of pairs)
constexpr size_t kCtrlBytes = 256;
// Compacted h rows of both models per token group of the sweeps' work order. Each of the B200's two
// L2 halves keeps its own copy of lines its SMs read, so the rows re-read for every vocabulary tile
// must fit in one half (~63 MB) beside the unembedding tiles in flight; measured best at 40 MB
// (32-56 MB tried: 40 gave the shortest steps on the long-context, large-vocabulary and spectral
// workloads; a workload whose rows fit in one group, like the OPD workload, is unaffected).
constexpr double kTokenGroupBytes = 40.0 * 1024 * 1024;

thread_local int g_launches = 0;
thread_local bool g_launch_failed = false;   // a launch of the current call was refused

// Opt-in per-kernel timing: events recorded on the launching stream around each launch.
struct TimingRec {
  int cat;
  cudaEvent_t a, b;
};
struct Timing {
  bool on = false;
  std::vector<TimingRec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
thread_local Timing g_timing;
thread_local int g_cat = NB_KL_KERNEL_ROWOPS;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

struct Layout {
  int64_t N, N_pad, V, d_s, d_t;
  int split;             // fp32 hidden states stored as [hi | lo] bf16
  int kb_s, kb_t;        // 64-wide K blocks of W
  int64_t lda_s, lda_t;  // row length of the compacted h buffers
  int n_vt, n_split;
  int n_big;             // forward sweeps: vocabulary units of kTilesPerUnitFwd tiles (the rest are single tiles)
  int64_t chunk_v;
  int n_chunks;          // backward vocabulary chunks
  size_t off_idx, off_inv, off_hs, off_ht, off_rl2s, off_rl2t, off_raux, off_rlab, off_labx, off_sched, off_dhc, off_state,
      off_part, off_G, g_bytes, total;
  long long fs_state;    // elements between state fields
};

// Vocabulary units of a sweep over n_vt tiles: the first (returned) units are runs of
// tiles_per_unit tiles, the rest single tiles, enough that the last ~kTailItems work items (over
// all n_tt token tiles) are short and the launch does not end on long items that leave most CTA
// pairs idle.
int big_units(int n_vt, int64_t n_tt, int tiles_per_unit) {
  const int n_single = int(std::min<int64_t>(n_vt, (kTailItems + n_tt - 1) / n_tt));
  return (n_vt - n_single) / tiles_per_unit;
}

bool make_layout(const nb_kl_shape* sh, float beta, Layout& L) {
  if (!sh) return false;
  if (sh->n_tokens < 0 || sh->vocab < 1 || sh->d_s < 8 || sh->d_t < 8) return false;
  if (sh->d_s % 8 || sh->d_t % 8) return false;
  if (sh->h_dtype != NB_BF16 && sh->h_dtype != NB_F32) return false;
  if (sh->reserved != 0) return false;
  if (sh->chunk_v < 0 || (sh->chunk_v % kBlockN) != 0) return false;
  if (sh->n_tokens > (int64_t(1) << 30) || sh->vocab > (int64_t(1) << 30) || sh->d_s > 65536 || sh->d_t > 65536)
    return false;
  L.N = sh->n_tokens;
  L.N_pad = round_up(std::max<int64_t>(L.N, 1), kPairM);
  L.V = sh->vocab;
  L.d_s = sh->d_s;
  L.d_t = sh->d_t;
  L.split = sh->h_dtype == NB_F32;
  L.kb_s = int((L.d_s + kBlockK - 1) / kBlockK);
  L.kb_t = int((L.d_t + kBlockK - 1) / kBlockK);
  L.lda_s = int64_t(L.kb_s) * kBlockK * (L.split ? 2 : 1);
  L.lda_t = int64_t(L.kb_t) * kBlockK * (L.split ? 2 : 1);
  L.n_vt = int((L.V + kBlockN - 1) / kBlockN);
  // forward units: runs of kTilesPerUnitFwd tiles, then single tiles
  L.n_big = big_units(L.n_vt, L.N_pad / kPairM, kTilesPerUnitFwd);
  L.n_split = 2 * (L.n_big + (L.n_vt - L.n_big * kTilesPerUnitFwd));  // two column halves per unit
  // default chunk: the vocabulary in equal chunks of at most ~24576 gradient tiles of 128 x 256
  // (the gradient buffer then takes at most ~1.5 GB whatever the token count; fewer, longer
  // chunks mean fewer launches and launch tails and fewer re-adds of the compacted dh
  // accumulator), but at least 4 d_s columns; at most 131072 columns
  if (sh->chunk_v) {
    L.chunk_v = sh->chunk_v;
  } else {
    const int64_t by_tiles = (int64_t(3) << 21) / (L.N_pad / kBlockM);
    const int64_t max_chunk = std::max<int64_t>(2048, std::min<int64_t>(131072, std::max<int64_t>(by_tiles, 4 * L.d_s)));
    const int64_t n_chunks = (L.V + max_chunk - 1) / max_chunk;
    L.chunk_v = round_up((L.V + n_chunks - 1) / n_chunks, kBlockN);
  }
  const bool jsd = beta > 0.f && beta < 1.f;
  size_t off = kCtrlBytes;
  L.off_idx = off;   off = align256(off + size_t(L.N_pad) * 4);
  L.off_inv = off;   off = align256(off + size_t(L.N_pad) * 4);   // compacted index of each position
  L.off_hs = off;    off = align256(off + size_t(L.N_pad) * L.lda_s * 2);
  L.off_ht = off;    off = align256(off + size_t(L.N_pad) * L.lda_t * 2);
  L.off_rl2s = off;  off = align256(off + size_t(L.N_pad) * 4);
  L.off_rl2t = off;  off = align256(off + size_t(L.N_pad) * 4);
  L.off_raux = off;  off = align256(off + size_t(L.N_pad) * 4);
  L.off_rlab = off;  off = align256(off + size_t(L.N_pad) * 4);   // label column per valid row
  L.off_labx = off;  off = align256(off + size_t(L.N_pad) * 4);   // student logit at the label
  L.n_chunks = int((L.V + L.chunk_v - 1) / L.chunk_v);
  L.off_sched = off; off = align256(off + size_t(2 * L.n_chunks + 2) * 4);   // one work counter per launch
  L.off_dhc = off;   off = align256(off + size_t(L.N_pad) * L.d_s * 4);        // compacted dh_s (backward)
  // the forward's split state and the backward's gradient-chunk buffer share one region
  const size_t state_bytes = align256(size_t(6) * L.n_split * L.N_pad * 4);
  const size_t part_bytes = jsd ? align256(size_t(2) * L.n_split * L.N_pad * 4) : 0;
  L.g_bytes = align256(size_t(L.N_pad) * L.chunk_v * 2);
  L.off_state = off;
  L.off_part = off + state_bytes;
  L.off_G = off;
  off += std::max(state_bytes + part_bytes, L.g_bytes);
  L.total = off;
  L.fs_state = (long long)L.n_split * L.N_pad;
  return true;
}

// ------------------------------------------------------------------ device / driver set-up
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

struct DevInfo {
  int sms = 0;
  int pairs = 0;         // CTA pairs (clusters of 2) that can be resident at once
  bool ok = false;
  bool attrs = false;
};

DevInfo g_dev[64];
std::mutex g_dev_mu;

nb_status device_info(DevInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NB_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.attrs) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return NB_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NB_ERR_CUDA;
    d.sms = sms;
    d.ok = major == 10;
    if (d.ok) {
      bool fail = false;
      fail |= cudaFuncSetAttribute(sweep_kernel<kStateNone>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kStateS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kStateT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kJsd>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kGradFkl>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kGradRkl>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(sweep_kernel<kGradJsd>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      fail |= cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess;
      if (fail) return NB_ERR_CUDA;
      // the warpgroup register split needs exactly the launch register count it was sized for
      const void* fns[] = {(const void*)sweep_kernel<kStateNone>, (const void*)sweep_kernel<kStateS>,
                           (const void*)sweep_kernel<kStateT>,    (const void*)sweep_kernel<kJsd>,
                           (const void*)sweep_kernel<kGradFkl>,   (const void*)sweep_kernel<kGradRkl>,
                           (const void*)sweep_kernel<kGradJsd>,   (const void*)gemm_kernel};
      for (const void* f : fns) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, f) != cudaSuccess) return NB_ERR_CUDA;
        if (fa.numRegs < kRegsLaunch) d.ok = false;
      }
      // persistent grids: as many pairs as fit at once (a cluster stays inside one GPC)
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (sms / 2));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, (const void*)sweep_kernel<kStateS>, &cfg) != cudaSuccess ||
          clusters < 1)
        clusters = sms / 2;
      d.pairs = std::min(clusters, sms / 2);
    }
    d.attrs = true;
  }
  out = d;
  return d.ok ? NB_OK : NB_ERR_UNSUPPORTED;
}

// 2-D tensor map; loads read out-of-range elements as zero, stores skip them.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 output map with 32 x 32 boxes (128-byte rows, 128-byte swizzle) for the GEMM epilogue
bool make_out_map(CUtensorMap* m, float* base, uint64_t cols, uint64_t rows) {
  return make_map(m, base, cols, rows, cols * 4, 32, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Every launch allows programmatic dependent launch: the kernel may start (and run its set-up)
// while the previous kernel in the stream finishes; its first global-memory access waits for that
// kernel (pdl_wait in every kernel). A failed launch is reported by check_launch().
template <typename... KArgs, typename... Args>
void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  TimingRec r{g_cat, nullptr, nullptr};
  if (g_timing.on) {
    r.a = g_timing.get();
    r.b = g_timing.get();
    cudaEventRecord(r.a, st);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) g_launch_failed = true;
  ++g_launches;
  if (g_timing.on) {
    cudaEventRecord(r.b, st);
    g_timing.recs.push_back(r);
  }
  g_cat = NB_KL_KERNEL_ROWOPS;
}

// the next launch belongs to category `c`
void next_cat(int c) { g_cat = c; }

nb_status check_launch() {
  const bool failed = g_launch_failed;
  g_launch_failed = false;
  return (cudaGetLastError() == cudaSuccess && !failed) ? NB_OK : NB_ERR_CUDA;
}

struct Ws {
  Ctrl* ctrl;
  int* idx;
  int* inv;
  int* sched;
  float* dhc;
  __nv_bfloat16 *hs, *ht;
  float *rl2s, *rl2t, *raux, *state, *part;
  int* rlab;
  float* labx;
  __nv_bfloat16* G;
};

Ws carve(const Layout& L, void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  Ws w;
  w.ctrl = reinterpret_cast<Ctrl*>(b);
  w.idx = reinterpret_cast<int*>(b + L.off_idx);
  w.inv = reinterpret_cast<int*>(b + L.off_inv);
  w.sched = reinterpret_cast<int*>(b + L.off_sched);
  w.dhc = reinterpret_cast<float*>(b + L.off_dhc);
  w.hs = reinterpret_cast<__nv_bfloat16*>(b + L.off_hs);
  w.ht = reinterpret_cast<__nv_bfloat16*>(b + L.off_ht);
  w.rl2s = reinterpret_cast<float*>(b + L.off_rl2s);
  w.rl2t = reinterpret_cast<float*>(b + L.off_rl2t);
  w.raux = reinterpret_cast<float*>(b + L.off_raux);
  w.rlab = reinterpret_cast<int*>(b + L.off_rlab);
  w.labx = reinterpret_cast<float*>(b + L.off_labx);
  w.state = reinterpret_cast<float*>(b + L.off_state);
  w.part = reinterpret_cast<float*>(b + L.off_part);
  w.G = reinterpret_cast<__nv_bfloat16*>(b + L.off_G);
  return w;
}

// The valid rows of both hidden states into the compacted bf16 buffers (one launch); with lse_s,
// also the per-row constants of the second pass and the backward.
void launch_gathers(const Layout& L, const Ws& w, const void* h_s, const void* h_t, cudaStream_t st,
                    const float* lse_s = nullptr, const float* lse_t = nullptr, const float* aux = nullptr) {
  const int div = L.split ? 2 : 1;
  const GatherSrc gs{h_s, int(L.d_s), int(L.lda_s), int(L.lda_s / div), w.hs};
  const GatherSrc gt{h_t, int(L.d_t), int(L.lda_t), int(L.lda_t / div), w.ht};
  float *r2s = nullptr, *r2t = nullptr, *rax = nullptr;
  if (lse_s) {
    r2s = w.rl2s;
    r2t = w.rl2t;
    rax = w.raux;
  }
  const dim3 grid(unsigned(L.N_pad), 2);
  if (L.split)
    launch(gather_rows_kernel<true>, grid, dim3(128), 0, st, gs, gt, (const int*)w.idx, (const Ctrl*)w.ctrl, lse_s,
           lse_t, aux, r2s, r2t, rax);
  else
    launch(gather_rows_kernel<false>, grid, dim3(128), 0, st, gs, gt, (const int*)w.idx, (const Ctrl*)w.ctrl, lse_s,
           lse_t, aux, r2s, r2t, rax);
}

bool sweep_maps(const Layout& L, const Ws& w, const void* W_s, const void* W_t, SweepMaps& m) {
  bool ok = true;
  ok &= make_map(&m.a_s, w.hs, L.lda_s, L.N_pad, L.lda_s * 2, kBlockK, kBlockM);
  ok &= make_map(&m.b_s, W_s, L.d_s, L.V, L.d_s * 2, kBlockK, kHalfB);  // each CTA: 128 W rows
  ok &= make_map(&m.a_t, w.ht, L.lda_t, L.N_pad, L.lda_t * 2, kBlockK, kBlockM);
  ok &= make_map(&m.b_t, W_t, L.d_t, L.V, L.d_t * 2, kBlockK, kHalfB);
  return ok;
}

SweepArgs base_sweep_args(const Layout& L, const Ws& w, float beta, float tau) {
  SweepArgs a;
  std::memset(&a, 0, sizeof(a));
  a.teacher_first = L.lda_t >= L.lda_s ? 1 : 0;
  a.V = int(L.V);
  a.v_begin = 0;
  a.v_end = int(L.V);
  a.nkb_s = int(L.lda_s / kBlockK);
  a.nkb_t = int(L.lda_t / kBlockK);
  a.bmod_s = L.kb_s;
  a.bmod_t = L.kb_t;
  a.tiles_per_unit = kTilesPerUnitFwd;
  a.n_big = L.n_big;
  a.scale = float(1.4426950408889634 / double(tau));
  a.beta = beta;
  a.ld = int(L.N_pad);
  a.field_stride = L.fs_state;
  a.row_l2s = w.rl2s;
  a.row_l2t = w.rl2t;
  a.row_aux = w.raux;
  a.n_valid = &w.ctrl->n_valid;
  a.gscale = &w.ctrl->gscale;
  a.status = &w.ctrl->status;
  a.wait_limit_ns = kWaitLimitNs;
  // token tiles per group: the group's compacted rows of both models within kTokenGroupBytes
  const double tile_bytes = double(kPairM) * double(L.lda_s + L.lda_t) * 2.0;
  a.tt_group = int(std::min(double(1 << 30), std::max(1.0, std::floor(kTokenGroupBytes / tile_bytes))));
  return a;
}

// grid of a pair kernel: 2 CTAs per pair, at most one resident wave of pairs
unsigned pair_grid(const DevInfo& dev, int work_items) {
  return unsigned(2 * std::max(1, std::min(dev.pairs, work_items)));
}

// Wide (256 x 512) GEMM tiles when they cover the N columns with no more padding than
// 256-wide tiles and still give every resident CTA pair a tile (`m_tiles`: 256-row tiles of
// the launch); their output column tile width.
int gemm_wide(int64_t N, int64_t m_tiles, int pairs) {
  if (round_up(N, 2 * kBlockN) != round_up(N, kBlockN)) return 0;
  return m_tiles * ((N + 2 * kBlockN - 1) / (2 * kBlockN)) >= pairs ? 1 : 0;
}
int gemm_tile_n(int wide) { return wide ? kWideN : kBlockN; }

int sweep_units(const Layout& L, const SweepArgs& a) {
  const int n_tt = int(L.N_pad / kPairM);
  const int n_vt = (a.v_end - a.v_begin + kBlockN - 1) / kBlockN;
  const int n_vu = a.n_big + (n_vt - a.n_big * a.tiles_per_unit);
  return n_tt * n_vu;
}

template <int MODE>
void launch_sweep(const DevInfo& dev, const Layout& L, const SweepMaps& m, const SweepArgs& a, cudaStream_t st) {
  next_cat(MODE <= kStateT ? NB_KL_KERNEL_SWEEP_FWD : MODE == kJsd ? NB_KL_KERNEL_SWEEP_JSD : NB_KL_KERNEL_SWEEP_GRAD);
  launch(sweep_kernel<MODE>, dim3(pair_grid(dev, sweep_units(L, a))), dim3(kThreads), size_t(kSmemBytes), st, m,
         a);
}

nb_status validate_common(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                          const void* W_t, const int64_t* labels, float beta, float tau, void* workspace,
                          size_t ws_bytes, Layout& L) {
  if (!make_layout(shape, beta, L)) return NB_ERR_INVALID_ARG;
  if (!(beta >= 0.f && beta <= 1.f)) return NB_ERR_INVALID_ARG;
  if (!(tau > 0.f) || !std::isfinite(tau)) return NB_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return NB_ERR_INVALID_ARG;
  if (L.N > 0) {
    if (!h_s || !W_s || !h_t || !W_t || !labels) return NB_ERR_INVALID_ARG;
    if (!aligned16(h_s) || !aligned16(W_s) || !aligned16(h_t) || !aligned16(W_t)) return NB_ERR_INVALID_ARG;
  }
  if (ws_bytes < L.total) return NB_ERR_WORKSPACE;
  return NB_OK;
}

// ------------------------------------------------------------------ fixed scratch
// Scratch of nb_kl_forward_noalloc: one array per device, created when the library's module
// is loaded on that device and kept until the process exits. Its device address is looked up
// once per device (with that device current) the first time the entry point runs there.
static __device__ __align__(256) uint8_t g_fixed_scratch[NB_KL_NOALLOC_SCRATCH_BYTES];

void* g_fixed_scratch_ptr[64] = {};
std::mutex g_fixed_mu;

nb_status fixed_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NB_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_fixed_mu);
  if (!g_fixed_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || p == nullptr) return NB_ERR_CUDA;
    g_fixed_scratch_ptr[dev] = p;
  }
  *out = g_fixed_scratch_ptr[dev];
  return NB_OK;
}

// Common start of the state-sweep forward calls: compaction of the valid rows (with the
// label column of each row relative to the vocabulary range [v_off, v_off + V) when `side`),
// bf16 gathers of both hidden states, the zeroed work counters and the sweep's tensor maps.
struct Prep {
  Layout L;
  Ws w;
  DevInfo dev;
  cudaStream_t st;
  SweepMaps maps;
  SweepArgs a;
};

nb_status prepare(Prep& P, const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                  const void* W_t, const int64_t* labels, float beta, float tau, int side, int64_t v_off,
                  int64_t* n_valid, void* workspace, cudaStream_t st) {
  const Layout& L = P.L;
  P.st = st;
  P.w = carve(L, workspace);
  const Ws& w = P.w;
  // all-ones bits are a NaN: a label column the sweep never meets leaves a NaN log-probability
  if (side && cudaMemsetAsync(w.labx, 0xFF, size_t(L.N_pad) * 4, st) != cudaSuccess) return NB_ERR_CUDA;
  // work counters zeroed first, so that the kernels of the call follow one another directly
  if (cudaMemsetAsync(w.sched, 0, size_t(2 * L.n_chunks + 2) * 4, st) != cudaSuccess) return NB_ERR_CUDA;
  launch(compact_kernel, dim3(1), dim3(kScanThreads), 0, st, labels, int(L.N), (long long)shape->ignore_index,
         w.idx, w.ctrl, n_valid, (const float*)nullptr, tau, side ? w.rlab : (int*)nullptr, (long long)L.V,
         (long long)v_off, (int*)nullptr);
  launch_gathers(L, w, h_s, h_t, st);
  if (!sweep_maps(L, w, W_s, W_t, P.maps)) return NB_ERR_CUDA;
  P.a = base_sweep_args(L, w, beta, tau);
  P.a.out = w.state;
  P.a.sched = w.sched;
  P.a.side = side;
  P.a.row_label = w.rlab;
  P.a.label_x = w.labx;
  return NB_OK;
}

// The state sweep of the method's direction; returns the merge's kl_dir.
int launch_state_sweep(const Prep& P, float beta) {
  if (beta == 1.f) {
    launch_sweep<kStateS>(P.dev, P.L, P.maps, P.a, P.st);
    return 1;
  }
  if (beta == 0.f) {
    launch_sweep<kStateT>(P.dev, P.L, P.maps, P.a, P.st);
    return 2;
  }
  launch_sweep<kStateNone>(P.dev, P.L, P.maps, P.a, P.st);
  return 0;
}

// Second JSD sweep (per-row base-2 LSEs already in row_l2s / row_l2t) and its reduction
// into out_js / out_ks [N] in nats.
void launch_jsd_pass(const Prep& P, float* out_js, float* out_ks) {
  SweepArgs b = P.a;
  b.side = 0;
  b.out = P.w.part;
  b.sched = P.w.sched + 1;
  launch_sweep<kJsd>(P.dev, P.L, P.maps, b, P.st);
  const unsigned rb = unsigned((P.L.N_pad + kMergeRows - 1) / kMergeRows);
  launch(jsd_finalize_kernel, dim3(rb), dim3(kMergeRows * kMergeLanes), 0, P.st, (const float*)P.w.part,
         (long long)P.L.fs_state, int(P.L.N_pad), P.L.n_split, (const int*)P.w.idx, (const Ctrl*)P.w.ctrl, out_js,
         out_ks);
}

void launch_merge(const Prep& P, int kl_dir, int side, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                  float* entropy_s, float* logp_label, float* vp_state) {
  const unsigned rb = unsigned((P.L.N_pad + kMergeRows - 1) / kMergeRows);
  launch(merge_kernel, dim3(rb), dim3(kMergeRows * kMergeLanes), 0, P.st, (const float*)P.w.state,
         (long long)P.L.fs_state, int(P.L.N_pad), P.L.n_split, (const int*)P.w.idx, (const Ctrl*)P.w.ctrl, kl_dir,
         loss_tok, lse_s, lse_t, aux, P.w.rl2s, P.w.rl2t, side, (const float*)P.w.labx, entropy_s, logp_label,
         vp_state, (long long)P.L.N);
}

nb_status zero_f32(float* p, int64_t n, cudaStream_t st) {
  return (!p || cudaMemsetAsync(p, 0, size_t(n) * 4, st) == cudaSuccess) ? NB_OK : NB_ERR_CUDA;
}

// One forward call; with `entropy_s` / `logp_label` (either may be null) the state sweep also
// produces the student's per-token side outputs.
nb_status forward_impl(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t, const void* W_t,
                       const int64_t* labels, float beta, float tau, float* loss_tok, float* lse_s, float* lse_t,
                       float* aux, float* loss_mean, int64_t* n_valid, float* entropy_s, float* logp_label,
                       void* workspace, size_t workspace_bytes, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  Prep P;
  nb_status s = validate_common(shape, h_s, W_s, h_t, W_t, labels, beta, tau, workspace, workspace_bytes, P.L);
  if (s != NB_OK) return s;
  const Layout& L = P.L;
  if (!loss_mean || !n_valid) return NB_ERR_INVALID_ARG;
  if (L.N > 0 && (!loss_tok || !lse_s || !lse_t || !aux)) return NB_ERR_INVALID_ARG;
  const int side = (entropy_s || logp_label) ? 1 : 0;
  if ((s = device_info(P.dev)) != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  if (L.N == 0) {
    if (cudaMemsetAsync(loss_mean, 0, sizeof(float), st) != cudaSuccess) return NB_ERR_CUDA;
    if (cudaMemsetAsync(n_valid, 0, sizeof(int64_t), st) != cudaSuccess) return NB_ERR_CUDA;
    return NB_OK;
  }
  for (float* o : {loss_tok, lse_s, lse_t, aux, entropy_s, logp_label})
    if ((s = zero_f32(o, L.N, st)) != NB_OK) return s;
  if ((s = prepare(P, shape, h_s, W_s, h_t, W_t, labels, beta, tau, side, 0, n_valid, workspace, st)) !=
      NB_OK)
    return s;
  const int kl_dir = launch_state_sweep(P, beta);
  launch_merge(P, kl_dir, side, loss_tok, lse_s, lse_t, aux, entropy_s, logp_label, nullptr);
  if (kl_dir == 0) launch_jsd_pass(P, loss_tok, aux);
  launch(mean_kernel, dim3(1), dim3(1024), 0, st, (const float*)loss_tok, int(L.N), (const Ctrl*)P.w.ctrl,
         loss_mean);
  return check_launch();
}

// Vocabulary-parallel forward, first part: this rank's shard of the vocabulary (rows
// [v_off, v_off + V) of the full unembeddings). Writes the shard's merged per-token state.
nb_status vp_state_impl(const nb_kl_shape* shape, int64_t v_off, const void* h_s, const void* W_s, const void* h_t,
                        const void* W_t, const int64_t* labels, float beta, float tau, float* state,
                        void* workspace, size_t workspace_bytes, cudaStream_t st) {
  g_launches = 0;
  g_launch_failed = false;
  Prep P;
  nb_status s = validate_common(shape, h_s, W_s, h_t, W_t, labels, beta, tau, workspace, workspace_bytes, P.L);
  if (s != NB_OK) return s;
  if (v_off < 0 || v_off > (int64_t(1) << 30)) return NB_ERR_INVALID_ARG;
  if (P.L.N > 0 && !state) return NB_ERR_INVALID_ARG;
  if ((s = device_info(P.dev)) != NB_OK) return s;
  if (cudaMemsetAsync(workspace, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  if (P.L.N == 0) return NB_OK;
  if ((s = zero_f32(state, int64_t(kVpFields) * P.L.N, st)) != NB_OK) return s;
  if ((s = prepare(P, shape, h_s, W_s, h_t, W_t, labels, beta, tau, 1, v_off, nullptr, workspace, st)) !=
      NB_OK)
    return s;
  const int kl_dir = launch_state_sweep(P, beta);
  launch_merge(P, kl_dir, 1, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, state);
  return check_launch();
}

// Vocabulary-parallel JSD, second sweep over this rank's shard with the global LSEs:
// per-token partial sums [2][N] in nats (the divergence and KL(S||M) over the shard).
nb_status vp_jsd_partial_impl(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                              const void* W_t, const int64_t* labels, float beta, float tau, const float* lse_s,
                              const float* lse_t, float* part, void* workspace, size_t workspace_bytes,
                              cudaStream_t st) {
  g_launches = 0;
  g_launch_failed = false;
  Prep P;
  nb_status s = validate_common(shape, h_s, W_s, h_t, W_t, labels, beta, tau, workspace, workspace_bytes, P.L);
  if (s != NB_OK) return s;
  if (!(beta > 0.f && beta < 1.f)) return NB_ERR_INVALID_ARG;
  if (P.L.N > 0 && (!lse_s || !lse_t || !part)) return NB_ERR_INVALID_ARG;
  if ((s = device_info(P.dev)) != NB_OK) return s;
  if (cudaMemsetAsync(workspace, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  if (P.L.N == 0) return NB_OK;
  if ((s = zero_f32(part, 2 * P.L.N, st)) != NB_OK) return s;
  P.st = st;
  P.w = carve(P.L, workspace);
  const Layout& L = P.L;
  const Ws& w = P.w;
  if (cudaMemsetAsync(w.sched, 0, size_t(2 * L.n_chunks + 2) * 4, st) != cudaSuccess) return NB_ERR_CUDA;
  launch(compact_kernel, dim3(1), dim3(kScanThreads), 0, st, labels, int(L.N), (long long)shape->ignore_index,
         w.idx, w.ctrl, (int64_t*)nullptr, (const float*)nullptr, tau, (int*)nullptr, (long long)L.V, 0ll,
         (int*)nullptr);
  // the global LSEs become the per-row base-2 constants of the second pass (aux is unused there)
  launch_gathers(L, w, h_s, h_t, st, lse_s, lse_t, lse_s);
  if (!sweep_maps(L, w, W_s, W_t, P.maps)) return NB_ERR_CUDA;
  P.a = base_sweep_args(L, w, beta, tau);
  P.a.sched = w.sched;
  launch_jsd_pass(P, part, part + L.N);
  return check_launch();
}

}  // namespace

// =====================================================================================
extern "C" {

size_t nb_kl_workspace_size(const nb_kl_shape* shape, float beta) {
  Layout L;
  if (!make_layout(shape, beta, L)) return 0;
  return L.total;
}

int64_t nb_kl_chunk_columns(const nb_kl_shape* shape) {
  Layout L;
  if (!make_layout(shape, 1.0f, L)) return 0;
  return L.chunk_v;
}

const char* nb_kl_status_string(nb_status s) {
  switch (s) {
    case NB_OK: return "ok";
    case NB_ERR_INVALID_ARG: return "invalid argument";
    case NB_ERR_UNSUPPORTED: return "unsupported device or size";
    case NB_ERR_WORKSPACE: return "workspace too small";
    case NB_ERR_CUDA: return "CUDA error";
    case NB_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int nb_kl_last_launch_count(void) { return g_launches; }

void nb_kl_timing_enable(int on) { g_timing.on = on != 0; }

int nb_kl_timing_read(double* ms, int* launches, int ncat) {
  if (ncat < 0) return -1;
  for (int i = 0; i < ncat; ++i) {
    if (ms) ms[i] = 0.0;
    if (launches) launches[i] = 0;
  }
  int n = 0;
  for (const TimingRec& r : g_timing.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess &&
        r.cat >= 0 && r.cat < ncat) {
      if (ms) ms[r.cat] += t;
      if (launches) launches[r.cat] += 1;
    }
    g_timing.pool.push_back(r.a);
    g_timing.pool.push_back(r.b);
    ++n;
  }
  g_timing.recs.clear();
  return n;
}

nb_status nb_kl_device_status(void* workspace, void* stream) {
  if (!workspace) return NB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int status = 0;
  if (cudaMemcpyAsync(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return NB_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return NB_ERR_CUDA;
  return static_cast<nb_status>(status);
}

nb_status nb_kl_forward(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                        const void* W_t, const int64_t* labels, float beta, float tau, float* loss_tok,
                        float* lse_s, float* lse_t, float* aux, float* loss_mean, int64_t* n_valid,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(shape, h_s, W_s, h_t, W_t, labels, beta, tau, loss_tok, lse_s, lse_t, aux, loss_mean, n_valid,
                      nullptr, nullptr, workspace, workspace_bytes, stream);
}

nb_status nb_kl_forward_side(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                             const void* W_t, const int64_t* labels, float beta, float tau, float* loss_tok,
                             float* lse_s, float* lse_t, float* aux, float* loss_mean, int64_t* n_valid,
                             float* entropy_s, float* logp_label, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return forward_impl(shape, h_s, W_s, h_t, W_t, labels, beta, tau, loss_tok, lse_s, lse_t, aux, loss_mean, n_valid,
                      entropy_s, logp_label, workspace, workspace_bytes, stream);
}

nb_status nb_kl_vp_state(const nb_kl_shape* shape, int64_t vocab_offset, const void* h_s, const void* W_s,
                         const void* h_t, const void* W_t, const int64_t* labels, float beta, float tau,
                         float* state, void* workspace, size_t workspace_bytes, void* stream) {
  return vp_state_impl(shape, vocab_offset, h_s, W_s, h_t, W_t, labels, beta, tau, state, workspace,
                       workspace_bytes, static_cast<cudaStream_t>(stream));
}

nb_status nb_kl_vp_combine(int64_t n_tokens, int n_parts, const float* states, const int64_t* labels,
                           int64_t ignore_index, float beta, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                           float* entropy_s, float* logp_label, float* loss_mean, int64_t* n_valid, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (n_tokens < 0 || n_tokens > (int64_t(1) << 30) || n_parts < 1 || n_parts > 4096) return NB_ERR_INVALID_ARG;
  if (!(beta >= 0.f && beta <= 1.f)) return NB_ERR_INVALID_ARG;
  if (!loss_mean || !n_valid) return NB_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!states || !labels || !loss_tok || !lse_s || !lse_t || !aux)) return NB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_tokens == 0) {
    if (cudaMemsetAsync(loss_mean, 0, sizeof(float), st) != cudaSuccess) return NB_ERR_CUDA;
    if (cudaMemsetAsync(n_valid, 0, sizeof(int64_t), st) != cudaSuccess) return NB_ERR_CUDA;
    return NB_OK;
  }
  const int kl_dir = beta == 1.f ? 1 : beta == 0.f ? 2 : 0;
  launch(vp_combine_kernel, dim3(unsigned((n_tokens + 127) / 128)), dim3(128), 0, st, states, n_parts,
         (long long)n_tokens, labels, (long long)ignore_index, kl_dir, loss_tok, lse_s, lse_t, aux, entropy_s,
         logp_label);
  launch(mean_count_kernel, dim3(1), dim3(1024), 0, st, (const float*)loss_tok, labels, (long long)n_tokens,
         (long long)ignore_index, loss_mean, n_valid);
  return check_launch();
}

nb_status nb_kl_vp_jsd_partial(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                               const void* W_t, const int64_t* labels, float beta, float tau, const float* lse_s,
                               const float* lse_t, float* part, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return vp_jsd_partial_impl(shape, h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, part, workspace,
                             workspace_bytes, static_cast<cudaStream_t>(stream));
}

nb_status nb_kl_vp_jsd_combine(int64_t n_tokens, int n_parts, const float* parts, const int64_t* labels,
                               int64_t ignore_index, float* loss_tok, float* aux, float* loss_mean, int64_t* n_valid,
                               void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (n_tokens < 0 || n_tokens > (int64_t(1) << 30) || n_parts < 1 || n_parts > 4096) return NB_ERR_INVALID_ARG;
  if (!loss_mean || !n_valid) return NB_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!parts || !labels || !loss_tok || !aux)) return NB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_tokens == 0) {
    if (cudaMemsetAsync(loss_mean, 0, sizeof(float), st) != cudaSuccess) return NB_ERR_CUDA;
    if (cudaMemsetAsync(n_valid, 0, sizeof(int64_t), st) != cudaSuccess) return NB_ERR_CUDA;
    return NB_OK;
  }
  launch(vp_jsd_combine_kernel, dim3(unsigned((n_tokens + 127) / 128)), dim3(128), 0, st, parts, n_parts,
         (long long)n_tokens, labels, (long long)ignore_index, loss_tok, aux);
  launch(mean_count_kernel, dim3(1), dim3(1024), 0, st, (const float*)loss_tok, labels, (long long)n_tokens,
         (long long)ignore_index, loss_mean, n_valid);
  return check_launch();
}

nb_status nb_kl_backward(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                         const void* W_t, const int64_t* labels, float beta, float tau, const float* lse_s,
                         const float* lse_t, const float* aux, const float* grad_out, float* dh_s, float* dW_s,
                         int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  Layout L;
  nb_status s = validate_common(shape, h_s, W_s, h_t, W_t, labels, beta, tau, workspace, workspace_bytes, L);
  if (s != NB_OK) return s;
  if (!dW_s || !grad_out) return NB_ERR_INVALID_ARG;
  if (!aligned16(dW_s)) return NB_ERR_INVALID_ARG;
  if (L.N > 0 && (!lse_s || !lse_t || !aux || !dh_s || !aligned16(dh_s))) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  if ((s = device_info(dev)) != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws w = carve(L, workspace);
  if (cudaMemsetAsync(w.ctrl, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  if (L.N == 0) {
    if (!accumulate_dW && cudaMemsetAsync(dW_s, 0, size_t(L.V) * L.d_s * 4, st) != cudaSuccess) return NB_ERR_CUDA;
    return NB_OK;
  }
  if (cudaMemsetAsync(w.sched, 0, size_t(2 * L.n_chunks + 2) * 4, st) != cudaSuccess) return NB_ERR_CUDA;
  launch(compact_kernel, dim3(1), dim3(kScanThreads), 0, st, labels, int(L.N), (long long)shape->ignore_index,
         w.idx, w.ctrl, (int64_t*)nullptr, grad_out, tau, (int*)nullptr, (long long)L.V, 0ll, w.inv);
  launch_gathers(L, w, h_s, h_t, st, lse_s, lse_t, aux);

  // one gradient-chunk buffer: per chunk the sweep writes it and the GEMMs then read it, in stream
  // order (two tensor-bound kernels gain nothing from overlapping; serial launches measured faster)
  SweepMaps maps;
  GemmMaps gm;
  bool ok = sweep_maps(L, w, W_s, W_t, maps);
  // gradient chunk written by the sweep epilogue: bf16 32 x 32 boxes, 64-byte rows
  ok &= make_map(&maps.g_out, w.G, L.chunk_v, L.N_pad, L.chunk_v * 2, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                 CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= make_out_map(&gm.out[0], w.dhc, L.d_s, L.N_pad);
  ok &= make_out_map(&gm.out[1], dW_s, L.d_s, L.V);
  // dh_s: A = G (K-major, box 64 x 128), B = W_s chunk as K x N (MN-major, 64 x 64 boxes)
  ok &= make_map(&gm.a[0], w.G, L.chunk_v, L.N_pad, L.chunk_v * 2, kBlockK, kBlockM);
  ok &= make_map(&gm.b[0], W_s, L.d_s, L.V, L.d_s * 2, 64, 64);
  // dW_s: A = G^T (MN-major), B = compacted h_s (hi part) as K x N (MN-major)
  ok &= make_map(&gm.a[1], w.G, L.chunk_v, L.N_pad, L.chunk_v * 2, 64, 64);
  ok &= make_map(&gm.b[1], w.hs, L.d_s, L.N_pad, L.lda_s * 2, 64, 64);
  if (!ok) return NB_ERR_CUDA;

  SweepArgs a = base_sweep_args(L, w, beta, tau);
  a.ldG = L.chunk_v;
  a.tiles_per_unit = kTilesPerUnitGrad;
  a.G = w.G;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.nprob = 2;
  // 256-row tiles of one chunk's launch: dh_s (tokens) and dW_s (chunk columns)
  g.wide = gemm_wide(L.d_s, L.N_pad / kPairM + (L.chunk_v + kPairM - 1) / kPairM, dev.pairs);
  g.n_valid = &w.ctrl->n_valid;
  g.status = &w.ctrl->status;
  g.wait_limit_ns = kWaitLimitNs;
  GemmProb& dh = g.prob[0];
  dh.a_mn = 0;
  dh.b_mn = 1;
  dh.m_dyn = 1;
  dh.N = int(L.d_s);
  dh.out_row0 = 0;
  GemmProb& dw = g.prob[1];
  dw.a_mn = 1;
  dw.b_mn = 1;
  dw.N = int(L.d_s);
  dw.k_dyn = 1;
  dw.accumulate = accumulate_dW ? 1 : 0;

  const int n_tt_max = int(L.N_pad / kPairM);
  const int n_dt = int((L.d_s + gemm_tile_n(g.wide) - 1) / gemm_tile_n(g.wide));   // output column tiles
  for (int c = 0; c < L.n_chunks; ++c) {
    const int64_t v0 = int64_t(c) * L.chunk_v, v1 = std::min(L.V, v0 + L.chunk_v);
    a.v_begin = int(v0);
    a.v_end = int(v1);
    a.n_big = big_units(int((v1 - v0 + kBlockN - 1) / kBlockN), L.N_pad / kPairM, kTilesPerUnitGrad);
    a.sched = w.sched + 2 * c;
    if (beta == 0.f) launch_sweep<kGradFkl>(dev, L, maps, a, st);
    else if (beta == 1.f) launch_sweep<kGradRkl>(dev, L, maps, a, st);
    else launch_sweep<kGradJsd>(dev, L, maps, a, st);
    dh.K = int(v1 - v0);
    dh.b_koff = int(v0);
    dh.accumulate = c > 0 ? 1 : 0;
    dw.M = int(v1 - v0);
    dw.out_row0 = int(v0);
    g.sched = w.sched + 2 * c + 1;
    const int tiles = n_tt_max * n_dt + int((v1 - v0 + kPairM - 1) / kPairM) * n_dt;
    next_cat(NB_KL_KERNEL_GEMM_BWD);
    launch(gemm_kernel, dim3(pair_grid(dev, tiles)), dim3(kThreads), size_t(kSmemBytes), st, gm, g);
  }
  // every row of dh_s: its compacted row, or zeros for a masked position
  launch(place_dh_kernel, dim3(unsigned(L.N)), dim3(128), 0, st, (const float*)w.dhc, int(L.d_s), dh_s,
         (const int*)w.inv);
  return check_launch();
}

nb_status nb_kl_forward_noalloc(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                                const void* W_t, const int64_t* labels, float beta, float tau, float* loss_tok,
                                float* lse_s, float* lse_t, float* aux, float* loss_mean, int64_t* n_valid,
                                void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  const size_t need = nb_kl_workspace_size(shape, beta);
  if (need == 0) return NB_ERR_INVALID_ARG;
  if (need > size_t(NB_KL_NOALLOC_SCRATCH_BYTES)) return NB_ERR_WORKSPACE;
  void* ws = nullptr;
  const nb_status s = fixed_scratch(&ws);
  if (s != NB_OK) return s;
  return nb_kl_forward(shape, h_s, W_s, h_t, W_t, labels, beta, tau, loss_tok, lse_s, lse_t, aux, loss_mean,
                       n_valid, ws, size_t(NB_KL_NOALLOC_SCRATCH_BYTES), stream);
}

nb_status nb_kl_noalloc_device_status(void* stream) {
  void* ws = nullptr;
  const nb_status s = fixed_scratch(&ws);
  if (s != NB_OK) return s;
  return nb_kl_device_status(ws, stream);
}

nb_status nb_kl_gram(const void* X, int64_t rows, int64_t d, float* G, void* workspace, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (!X || !G || !workspace) return NB_ERR_INVALID_ARG;
  if (rows < 1 || d < 8 || d % 8 || rows > (int64_t(1) << 30) || d > 65536) return NB_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(G) || !aligned16(workspace)) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ctrl* ctrl = static_cast<Ctrl*>(workspace);
  if (cudaMemsetAsync(ctrl, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  GemmMaps gm;
  std::memset(&gm, 0, sizeof(gm));
  // A = X^T (M = d contiguous) and B = X as K x N: both MN-major views of X's rows
  bool ok = make_map(&gm.a[0], X, uint64_t(d), uint64_t(rows), uint64_t(d) * 2, 64, 64);
  ok &= make_map(&gm.b[0], X, uint64_t(d), uint64_t(rows), uint64_t(d) * 2, 64, 64);
  ok &= make_out_map(&gm.out[0], G, uint64_t(d), uint64_t(d));
  if (!ok) return NB_ERR_CUDA;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.nprob = 1;
  g.n_valid = &ctrl->n_valid;
  g.status = &ctrl->status;
  g.wait_limit_ns = kWaitLimitNs;
  GemmProb& q = g.prob[0];
  q.a_mn = 1;
  q.b_mn = 1;
  q.M = int(d);
  q.N = int(d);
  q.K = int(rows);
  g.wide = gemm_wide(d, (d + kPairM - 1) / kPairM, dev.pairs);
  const int tiles = int((d + kPairM - 1) / kPairM * ((d + gemm_tile_n(g.wide) - 1) / gemm_tile_n(g.wide)));
  next_cat(NB_KL_KERNEL_GEMM_PROJ);
  launch(gemm_kernel, dim3(pair_grid(dev, tiles)), dim3(kThreads), size_t(kSmemBytes), st, gm, g);
  return check_launch();
}

nb_status nb_kl_project(const void* X, int64_t rows, int64_t d, const void* B, int64_t k, void* Y, void* workspace,
                        void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (!X || !B || !Y || !workspace) return NB_ERR_INVALID_ARG;
  if (rows < 1 || d < 8 || k < 8 || d % 8 || k % 8) return NB_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 30) || d > 65536 || k > 65536) return NB_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(B) || !aligned16(Y) || !aligned16(workspace)) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ctrl* ctrl = static_cast<Ctrl*>(workspace);
  if (cudaMemsetAsync(ctrl, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  GemmMaps gm;
  std::memset(&gm, 0, sizeof(gm));
  // A = X (K-major rows), B = the basis [d][k] as K x N (MN-major), out = Y [rows][k] bf16
  bool ok = make_map(&gm.a[0], X, uint64_t(d), uint64_t(rows), uint64_t(d) * 2, kBlockK, kBlockM);
  ok &= make_map(&gm.b[0], B, uint64_t(k), uint64_t(d), uint64_t(k) * 2, 64, 64);
  ok &= make_map(&gm.out[0], Y, uint64_t(k), uint64_t(rows), uint64_t(k) * 2, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                 CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) return NB_ERR_CUDA;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.nprob = 1;
  g.n_valid = &ctrl->n_valid;
  g.status = &ctrl->status;
  g.wait_limit_ns = kWaitLimitNs;
  GemmProb& q = g.prob[0];
  q.a_mn = 0;
  q.b_mn = 1;
  q.M = int(rows);
  q.N = int(k);
  q.K = int(d);
  q.out_bf16 = 1;
  g.wide = gemm_wide(k, (rows + kPairM - 1) / kPairM, dev.pairs);
  const int tiles = int((rows + kPairM - 1) / kPairM * ((k + gemm_tile_n(g.wide) - 1) / gemm_tile_n(g.wide)));
  next_cat(NB_KL_KERNEL_GEMM_PROJ);
  launch(gemm_kernel, dim3(pair_grid(dev, tiles)), dim3(kThreads), size_t(kSmemBytes), st, gm, g);
  return check_launch();
}

nb_status nb_kl_spectral_select(const double* evals, const double* evecs, int64_t d, int64_t k, void* V_k,
                                double* sigma, double* V_k_f64, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (!evals || !evecs || !V_k || !sigma) return NB_ERR_INVALID_ARG;
  if (d < 1 || d > 65536 || k < 1 || k > d) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  next_cat(NB_KL_KERNEL_GEMM_PROJ);
  launch(spectral_select_kernel, dim3(unsigned(d)), dim3(256), 0, static_cast<cudaStream_t>(stream), evals, evecs,
         int(d), int(k), static_cast<__nv_bfloat16*>(V_k), V_k_f64, sigma);
  return check_launch();
}

nb_status nb_kl_handoff_rows(const void* src, void* dst, int64_t n_rows, int64_t row_bytes, const int64_t* labels,
                             int64_t ignore_index, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (n_rows < 0 || row_bytes < 16 || row_bytes % 16 || row_bytes > (int64_t(1) << 24)) return NB_ERR_INVALID_ARG;
  if (n_rows == 0) return NB_OK;
  if (!src || !dst || !aligned16(src) || !aligned16(dst)) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  // two resident 256-thread blocks per SM; fewer when there are fewer rows than warps
  const long long warps = std::min<long long>(n_rows, 16ll * dev.sms);
  const unsigned blocks = unsigned((warps + 7) / 8);
  next_cat(NB_KL_KERNEL_HANDOFF);
  launch(handoff_rows_kernel, dim3(blocks), dim3(256), 0, static_cast<cudaStream_t>(stream),
         static_cast<const uint4*>(src), static_cast<uint4*>(dst), (long long)n_rows, (long long)(row_bytes / 16),
         labels, (long long)ignore_index);
  return check_launch();
}

nb_status nb_kl_enable_peer_access(int peer_device) {
  int dev = 0, can = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NB_ERR_CUDA;
  if (peer_device == dev) return NB_OK;
  if (cudaDeviceCanAccessPeer(&can, dev, peer_device) != cudaSuccess) return NB_ERR_INVALID_ARG;
  if (!can) return NB_ERR_UNSUPPORTED;
  const cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
  if (e == cudaErrorPeerAccessAlreadyEnabled) {
    cudaGetLastError();   // the call also recorded it as the last error: clear that
    return NB_OK;
  }
  return e == cudaSuccess ? NB_OK : NB_ERR_CUDA;
}

nb_status nb_kl_debug_gemm(const void* A, int a_mn_major, const void* B, int b_mn_major, int64_t M, int64_t N,
                           int64_t K, float* C, void* workspace, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (!A || !B || !C || !workspace) return NB_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || M % 8 || N % 8 || K % 8) return NB_ERR_INVALID_ARG;
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return NB_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || !aligned16(workspace)) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ctrl* ctrl = static_cast<Ctrl*>(workspace);
  if (cudaMemsetAsync(ctrl, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  GemmMaps gm;
  std::memset(&gm, 0, sizeof(gm));
  bool ok = true;
  if (!a_mn_major) ok &= make_map(&gm.a[0], A, K, M, K * 2, kBlockK, kBlockM);
  else ok &= make_map(&gm.a[0], A, M, K, M * 2, 64, 64);
  if (!b_mn_major) ok &= make_map(&gm.b[0], B, K, N, K * 2, kBlockK, kHalfB);
  else ok &= make_map(&gm.b[0], B, N, K, N * 2, 64, 64);
  if (!ok) return NB_ERR_CUDA;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.nprob = 1;
  g.n_valid = &ctrl->n_valid;
  g.status = &ctrl->status;
  g.wait_limit_ns = kWaitLimitNs;
  GemmProb& q = g.prob[0];
  q.a_mn = a_mn_major ? 1 : 0;
  q.b_mn = b_mn_major ? 1 : 0;
  q.M = int(M);
  q.N = int(N);
  q.K = int(K);
  ok = make_out_map(&gm.out[0], C, N, M);
  if (!ok) return NB_ERR_CUDA;
  g.wide = gemm_wide(N, (M + kPairM - 1) / kPairM, dev.pairs);
  const int tiles = int((M + kPairM - 1) / kPairM * ((N + gemm_tile_n(g.wide) - 1) / gemm_tile_n(g.wide)));
  launch(gemm_kernel, dim3(pair_grid(dev, tiles)), dim3(kThreads), size_t(kSmemBytes), st, gm, g);
  return check_launch();
}

nb_status nb_kl_debug_wait_timeout(void* workspace, uint64_t limit_ns, int sleeping, void* stream) {
  g_launches = 0;
  g_launch_failed = false;
  if (!workspace || !aligned16(workspace)) return NB_ERR_INVALID_ARG;
  if (limit_ns > 5000000000ull) return NB_ERR_INVALID_ARG;
  DevInfo dev;
  nb_status s = device_info(dev);
  if (s != NB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kCtrlBytes, st) != cudaSuccess) return NB_ERR_CUDA;
  launch(wait_timeout_kernel, dim3(1), dim3(32), 0, st, &static_cast<Ctrl*>(workspace)->status,
         (unsigned long long)limit_ns, sleeping ? 1 : 0);
  return check_launch();
}

}  // extern "C"
