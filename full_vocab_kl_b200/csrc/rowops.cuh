// Per-row kernels around the sweeps: valid-row compaction, the split-V LSE merge,
// the per-token finalisation and the masked per-token mean.
//
// "03 White-box OPD", section 2.3: keep the positions whose label is not -100 and
// divide the summed per-token divergence by their count (a per-token mean).
#pragma once

#include "common.cuh"

namespace nbkl {

struct Ctrl {          // first bytes of every workspace
  int status;          // device status word (0 = ok)
  int n_valid;         // number of rows with label != ignore_index
  float gscale;        // grad_out / (n_valid * tau), backward only
  int pad[61];
};

// ------------------------------------------------------------------ compaction (one block)
// Stable list of valid rows: idx[i] = position of the i-th label != ignore_index.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) compact_kernel(const int64_t* __restrict__ labels, int N,
                                                               long long ignore_index, int* __restrict__ idx,
                                                               Ctrl* ctrl, int64_t* n_valid_out,
                                                               const float* grad_out, float tau) {
  __shared__ int warp_sums[32];
  __shared__ int s_total;
  const int per = (N + kScanThreads - 1) / kScanThreads;
  const int b = threadIdx.x * per, e = min(N, b + per);
  int cnt = 0;
  for (int i = b; i < e; ++i) cnt += (labels[i] != ignore_index);
  // block exclusive scan of cnt
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
    int wi = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - ws;
    if (lane == 31) s_total = wi;
  }
  __syncthreads();
  int pos = warp_sums[warp] + incl - cnt;
  for (int i = b; i < e; ++i)
    if (labels[i] != ignore_index) idx[pos++] = i;
  if (threadIdx.x == 0) {
    const int nv = s_total;
    ctrl->n_valid = nv;
    if (n_valid_out) *n_valid_out = nv;
    if (grad_out) ctrl->gscale = nv > 0 ? grad_out[0] / (float(nv) * tau) : 0.f;
  }
}

// ------------------------------------------------------------------ gather of valid rows
// dst row i (< n_valid) = src row idx[i] as bf16, zero-padded to `lda` columns; rows
// n_valid .. round_up(n_valid, 256) (the last pair tile) are zeroed. With `split`, an fp32 source is stored as
// [hi | lo] with hi = bf16(x) and lo = bf16(x - hi), each half `half` columns wide, so that
// hi*W + lo*W carries x to about 16 bits.
template <bool F32_SRC>
__global__ void gather_rows_kernel(const void* __restrict__ src, int d, __nv_bfloat16* __restrict__ dst, int lda,
                                   int half, const int* __restrict__ idx, const Ctrl* __restrict__ ctrl,
                                   // optional per-row constants (backward): base-2 LSEs and aux
                                   const float* lse_s, const float* lse_t, const float* aux, float* row_l2s,
                                   float* row_l2t, float* row_aux) {
  const int i = blockIdx.x;
  const int nv = ctrl->n_valid;
  const int rows_needed = ((nv + kPairM - 1) / kPairM) * kPairM;
  if (i >= rows_needed) return;
  __nv_bfloat16* out = dst + (long long)i * lda;
  const bool live = i < nv;
  const int r = live ? idx[i] : 0;
  if (row_l2s && threadIdx.x == 0) {
    row_l2s[i] = live ? lse_s[r] * kLog2e : 0.f;
    row_l2t[i] = live ? lse_t[r] * kLog2e : 0.f;
    row_aux[i] = live ? aux[r] : 0.f;
  }
  if (!F32_SRC) {
    const __nv_bfloat16* in = static_cast<const __nv_bfloat16*>(src) + (long long)r * d;
    // d is a multiple of 8: 16-byte vectors
    for (int c = threadIdx.x * 8; c < lda; c += blockDim.x * 8) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (live && c < d) v = *reinterpret_cast<const uint4*>(in + c);
      *reinterpret_cast<uint4*>(out + c) = v;
    }
  } else {
    const float* in = static_cast<const float*>(src) + (long long)r * d;
    for (int c = threadIdx.x; c < half; c += blockDim.x) {
      float x = (live && c < d) ? in[c] : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      out[c] = hi;
      out[half + c] = lo;
    }
  }
}

// ------------------------------------------------------------------ split-V merge
// Merge the per-split online states of every valid row (max-rescaled sums) and write
// the natural-log LSEs and, for the KL directions, the per-token loss.
//   LSE(u) = ln 2 * (m + log2 l),  KL = ln 2 * (a / l_p - L2_p + L2_q)
// `kl_dir`: 1 reverse (p = student), 2 forward (p = teacher), 0 none (JSD pass 1: the
// base-2 LSEs go to row_l2s / row_l2t for the second pass).
// Block = 32 rows x 8 split lanes: lane j of row r visits splits j, j + 8, ... so that a warp
// (32 consecutive rows, one split) reads contiguous memory; the 8 partial results of a row
// are combined in shared memory in a fixed order.
constexpr int kMergeRows = 32, kMergeLanes = 8;

__global__ void __launch_bounds__(kMergeRows * kMergeLanes)
    merge_kernel(const float* __restrict__ state, long long fs, int ld, int n_split, const int* __restrict__ idx,
                 const Ctrl* __restrict__ ctrl, int kl_dir, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                 float* row_l2s, float* row_l2t) {
  __shared__ float sm_s[kMergeLanes][kMergeRows], sm_t[kMergeLanes][kMergeRows];
  __shared__ double sl_s[kMergeLanes][kMergeRows], sl_t[kMergeLanes][kMergeRows], sa[kMergeLanes][kMergeRows];
  const int r = threadIdx.x % kMergeRows, j = threadIdx.x / kMergeRows;
  const int nv = ctrl->n_valid;
  const int i = blockIdx.x * kMergeRows + r;
  const bool live = i < nv;
  float ms = kNegBig, mt = kNegBig;
  if (live)
    for (int k = j; k < n_split; k += kMergeLanes) {
      ms = fmaxf(ms, state[(long long)k * ld + i]);
      mt = fmaxf(mt, state[2 * fs + (long long)k * ld + i]);
    }
  sm_s[j][r] = ms;
  sm_t[j][r] = mt;
  __syncthreads();
  ms = kNegBig;
  mt = kNegBig;
  for (int q = 0; q < kMergeLanes; ++q) {
    ms = fmaxf(ms, sm_s[q][r]);
    mt = fmaxf(mt, sm_t[q][r]);
  }
  double ls = 0.0, lt = 0.0, a = 0.0;
  if (live)
    for (int k = j; k < n_split; k += kMergeLanes) {
      const long long o = (long long)k * ld + i;
      const double fs_ = exp2f(state[o] - ms);
      const double ft_ = exp2f(state[2 * fs + o] - mt);
      ls += state[fs + o] * fs_;
      lt += state[3 * fs + o] * ft_;
      if (kl_dir == 1) a += state[4 * fs + o] * fs_;
      if (kl_dir == 2) a += state[4 * fs + o] * ft_;
    }
  sl_s[j][r] = ls;
  sl_t[j][r] = lt;
  sa[j][r] = a;
  __syncthreads();
  if (j != 0 || !live) return;
  ls = lt = a = 0.0;
  for (int q = 0; q < kMergeLanes; ++q) {
    ls += sl_s[q][r];
    lt += sl_t[q][r];
    a += sa[q][r];
  }
  const double L2s = ms + log2(ls), L2t = mt + log2(lt);
  const int row = idx[i];
  lse_s[row] = float(L2s * 0.69314718055994530942);
  lse_t[row] = float(L2t * 0.69314718055994530942);
  if (kl_dir == 1) {
    const float kl = float(0.69314718055994530942 * (a / ls - L2s + L2t));
    loss_tok[row] = kl;
    aux[row] = kl;
  } else if (kl_dir == 2) {
    const float kl = float(0.69314718055994530942 * (a / lt - L2t + L2s));
    loss_tok[row] = kl;
    aux[row] = kl;
  } else {
    row_l2s[i] = float(L2s);
    row_l2t[i] = float(L2t);
  }
}

// JSD: sum the per-split partial sums (base 2) in a fixed order and convert to nats.
__global__ void __launch_bounds__(kMergeRows * kMergeLanes)
    jsd_finalize_kernel(const float* __restrict__ part, long long fs, int ld, int n_split,
                        const int* __restrict__ idx, const Ctrl* __restrict__ ctrl, float* loss_tok, float* aux) {
  __shared__ double sj[kMergeLanes][kMergeRows], sk[kMergeLanes][kMergeRows];
  const int r = threadIdx.x % kMergeRows, j = threadIdx.x / kMergeRows;
  const int nv = ctrl->n_valid;
  const int i = blockIdx.x * kMergeRows + r;
  const bool live = i < nv;
  double js = 0.0, ks = 0.0;
  if (live)
    for (int k = j; k < n_split; k += kMergeLanes) {
      js += part[(long long)k * ld + i];
      ks += part[fs + (long long)k * ld + i];
    }
  sj[j][r] = js;
  sk[j][r] = ks;
  __syncthreads();
  if (j != 0 || !live) return;
  js = ks = 0.0;
  for (int q = 0; q < kMergeLanes; ++q) {
    js += sj[q][r];
    ks += sk[q][r];
  }
  const int row = idx[i];
  loss_tok[row] = float(js * 0.69314718055994530942);
  aux[row] = float(ks * 0.69314718055994530942);
}

// Deterministic masked mean: fixed-order fp64 sum of loss_tok (masked rows hold 0).
__global__ void __launch_bounds__(1024) mean_kernel(const float* __restrict__ loss_tok, int N,
                                                    const Ctrl* __restrict__ ctrl, float* loss_mean) {
  __shared__ double part[1024];
  double s = 0.0;
  for (int i = threadIdx.x; i < N; i += 1024) s += loss_tok[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int nv = ctrl->n_valid;
    *loss_mean = nv > 0 ? float(part[0] / nv) : 0.f;
  }
}

// dh_s[idx[i]] = dh_c[i] for the valid rows (the GEMMs accumulate into the compacted dh_c).
__global__ void scatter_rows_kernel(const float* __restrict__ src, int d, float* __restrict__ dst,
                                    const int* __restrict__ idx, const Ctrl* __restrict__ ctrl) {
  const int i = blockIdx.x;
  if (i >= ctrl->n_valid) return;
  const float4* in = reinterpret_cast<const float4*>(src + (long long)i * d);
  float4* out = reinterpret_cast<float4*>(dst + (long long)idx[i] * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) out[c] = in[c];
}

// Zero the dh_s rows of masked positions (valid rows are written by the scatter).
__global__ void zero_masked_rows_kernel(const int64_t* __restrict__ labels, long long ignore_index, float* dh,
                                        int d) {
  const int r = blockIdx.x;
  if (labels[r] != ignore_index) return;
  float* row = dh + (long long)r * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) row[c] = 0.f;
}

// Test hook: wait on an mbarrier that nothing arrives at, with the given limit.
__global__ void wait_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl w{status, limit_ns};
    mbar_wait(&bar, 0, w);
  }
}

}  // namespace nbkl
