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
// Stable list of valid rows: idx[i] = position of the i-th label != ignore_index. Each of the
// 32 warps owns one contiguous segment of the labels and reads it in coalesced runs of 32: a
// count pass (warp ballots), a scan of the 32 segment counts, a placement pass. With
// `row_label`, also the label of each valid row as a column of the vocabulary range
// [v_off, v_off + V) held here (-1 outside it); with `inv`, the compacted index of every
// position (-1 for a masked one).
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) compact_kernel(const int64_t* __restrict__ labels, int N,
                                                               long long ignore_index, int* __restrict__ idx,
                                                               Ctrl* ctrl, int64_t* n_valid_out,
                                                               const float* grad_out, float tau,
                                                               int* __restrict__ row_label, long long V,
                                                               long long v_off, int* __restrict__ inv) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int warp_off[32];
  __shared__ int s_total;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = ((N + 31) / 32 + 31) & ~31;   // labels per warp, a multiple of 32
  const int b = min(N, warp * seg), e = min(N, b + seg);
  int cnt = 0;
  for (int base = b; base < e; base += 32) {
    const int i = base + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, i < e && labels[i] != ignore_index));
  }
  if (lane == 0) warp_off[warp] = cnt;
  __syncthreads();
  if (warp == 0) {   // exclusive scan of the 32 segment counts
    const int c = warp_off[lane];
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    warp_off[lane] = incl - c;
    if (lane == 31) s_total = incl;
  }
  __syncthreads();
  int pos = warp_off[warp];
  for (int base = b; base < e; base += 32) {
    const int i = base + lane;
    const long long y = i < e ? labels[i] : ignore_index;
    const bool v = i < e && y != ignore_index;
    const unsigned m = __ballot_sync(0xffffffffu, v);
    const int p = pos + __popc(m & ((1u << lane) - 1u));
    if (v) {
      idx[p] = i;
      if (row_label) row_label[p] = (y >= v_off && y - v_off < V) ? int(y - v_off) : -1;
    }
    if (inv && i < e) inv[i] = v ? p : -1;
    pos += __popc(m);
  }
  if (threadIdx.x == 0) {
    const int nv = s_total;
    ctrl->n_valid = nv;
    if (n_valid_out) *n_valid_out = nv;
    if (grad_out) ctrl->gscale = nv > 0 ? grad_out[0] / (float(nv) * tau) : 0.f;
  }
}

// ------------------------------------------------------------------ gather of valid rows
// Both models in one launch (blockIdx.y: 0 student, 1 teacher). dst row i (< n_valid) = src row
// idx[i] as bf16, zero-padded to `lda` columns; rows n_valid .. round_up(n_valid, 256) (the last
// pair tile) are zeroed. With `split`, an fp32 source is stored as [hi | lo] with hi = bf16(x) and
// lo = bf16(x - hi), each half `half` columns wide, so that hi*W + lo*W carries x to about 16 bits.
struct GatherSrc {
  const void* src;
  int d, lda, half;
  __nv_bfloat16* dst;
};

template <bool F32_SRC>
__global__ void gather_rows_kernel(GatherSrc g0, GatherSrc g1, const int* __restrict__ idx,
                                   const Ctrl* __restrict__ ctrl,
                                   // optional per-row constants (backward): base-2 LSEs and aux
                                   const float* lse_s, const float* lse_t, const float* aux, float* row_l2s,
                                   float* row_l2t, float* row_aux) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x;
  const int nv = ctrl->n_valid;
  const int rows_needed = ((nv + kPairM - 1) / kPairM) * kPairM;
  if (i >= rows_needed) return;
  const GatherSrc g = blockIdx.y ? g1 : g0;
  __nv_bfloat16* out = g.dst + (long long)i * g.lda;
  const bool live = i < nv;
  const int r = live ? idx[i] : 0;
  if (row_l2s && blockIdx.y == 0 && threadIdx.x == 0) {
    row_l2s[i] = live ? lse_s[r] * kLog2e : 0.f;
    row_l2t[i] = live ? lse_t[r] * kLog2e : 0.f;
    row_aux[i] = live ? aux[r] : 0.f;
  }
  if (!F32_SRC) {
    const __nv_bfloat16* in = static_cast<const __nv_bfloat16*>(g.src) + (long long)r * g.d;
    // d is a multiple of 8: 16-byte vectors
    for (int c = threadIdx.x * 8; c < g.lda; c += blockDim.x * 8) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (live && c < g.d) v = *reinterpret_cast<const uint4*>(in + c);
      *reinterpret_cast<uint4*>(out + c) = v;
    }
  } else {
    const float* in = static_cast<const float*>(g.src) + (long long)r * g.d;
    for (int c = threadIdx.x; c < g.half; c += blockDim.x) {
      float x = (live && c < g.d) ? in[c] : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      out[c] = hi;
      out[g.half + c] = lo;
    }
  }
}

// ------------------------------------------------------------------ split-V merge
// Merge the per-split online states of every valid row (max-rescaled sums) and write
// the natural-log LSEs and, for the KL directions, the per-token loss.
//   LSE(u) = ln 2 * (m + log2 l),  KL = ln 2 * (a / l_p - L2_p + L2_q)
// `kl_dir`: 1 reverse (p = student), 2 forward (p = teacher), 0 none (JSD pass 1: the
// base-2 LSEs go to row_l2s / row_l2t for the second pass).
// With `side`, the student's entropy and label log-probability are written as well:
//   H = ln 2 * (log2 l_s - E / l_s), E = sum_k 2^(m_k - M) (e_k + (m_k - M) l_k)
//   log S[label] = ln 2 * (x_label - L2_s)  (NaN when the sweep saw no label column)
// Block = 32 rows x 16 split lanes: lane j of row r visits splits j, j + 16, ... so that a warp
// (32 consecutive rows, one split) reads contiguous memory; the 16 partial results of a row
// are combined in shared memory in a fixed order.
constexpr int kMergeRows = 32, kMergeLanes = 16;

__global__ void __launch_bounds__(kMergeRows * kMergeLanes)
    merge_kernel(const float* __restrict__ state, long long fs, int ld, int n_split, const int* __restrict__ idx,
                 const Ctrl* __restrict__ ctrl, int kl_dir, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                 float* row_l2s, float* row_l2t, int side, const float* __restrict__ label_x, float* entropy_s,
                 float* logp_label, float* vp_state, long long vp_ld) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float sm_s[kMergeLanes][kMergeRows], sm_t[kMergeLanes][kMergeRows];
  __shared__ double sl_s[kMergeLanes][kMergeRows], sl_t[kMergeLanes][kMergeRows], sa[kMergeLanes][kMergeRows];
  __shared__ double se[kMergeLanes][kMergeRows];
  const int r = threadIdx.x % kMergeRows, j = threadIdx.x / kMergeRows;
  const int nv = ctrl->n_valid;
  const int i = blockIdx.x * kMergeRows + r;
  const bool live = i < nv;
  float ms = kNegBig, mt = kNegBig;
  if (live)
#pragma unroll 2
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
  double ls = 0.0, lt = 0.0, a = 0.0, e = 0.0;
  if (live)
#pragma unroll 2
    for (int k = j; k < n_split; k += kMergeLanes) {
      const long long o = (long long)k * ld + i;
      const double fs_ = exp2f(state[o] - ms);
      const double ft_ = exp2f(state[2 * fs + o] - mt);
      ls += state[fs + o] * fs_;
      lt += state[3 * fs + o] * ft_;
      if (kl_dir == 1) a += state[4 * fs + o] * fs_;
      if (kl_dir == 2) a += state[4 * fs + o] * ft_;
      if (side) e += (double(state[5 * fs + o]) + (double(state[o]) - ms) * state[fs + o]) * fs_;
    }
  sl_s[j][r] = ls;
  sl_t[j][r] = lt;
  sa[j][r] = a;
  se[j][r] = e;
  __syncthreads();
  if (j != 0 || !live) return;
  ls = lt = a = e = 0.0;
  for (int q = 0; q < kMergeLanes; ++q) {
    ls += sl_s[q][r];
    lt += sl_t[q][r];
    a += sa[q][r];
    e += se[q][r];
  }
  const int row = idx[i];
  if (vp_state) {   // one vocabulary shard: its merged state, finished by vp_combine_kernel
    vp_state[row] = ms;
    vp_state[vp_ld + row] = float(ls);
    vp_state[2 * vp_ld + row] = mt;
    vp_state[3 * vp_ld + row] = float(lt);
    vp_state[4 * vp_ld + row] = float(a);
    vp_state[5 * vp_ld + row] = float(e);
    vp_state[6 * vp_ld + row] = side ? label_x[i] : __int_as_float(0x7fffffff);
    return;
  }
  const double L2s = ms + log2(ls), L2t = mt + log2(lt);
  lse_s[row] = float(L2s * 0.69314718055994530942);
  lse_t[row] = float(L2t * 0.69314718055994530942);
  if (side) {
    if (entropy_s) entropy_s[row] = float(0.69314718055994530942 * (log2(ls) - e / ls));
    if (logp_label) logp_label[row] = float(0.69314718055994530942 * (double(label_x[i]) - L2s));
  }
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
  pdl_wait();
  pdl_launch_dependents();
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

// ------------------------------------------------------------------ vocabulary-parallel combine
// Exchange format of one vocabulary shard, field-major [kVpFields][n_tokens] fp32, base-2
// tempered units (x = u log2 e): m_s, l_s, m_t, l_t, a, e (see merge_kernel) and the student
// logit at the row's label (NaN when the label is not in the shard).
constexpr int kVpFields = 7;

// Merge the states of `n_parts` shards ([part][field][n_tokens], fixed part order, fp64
// sums) and finish each valid row exactly as merge_kernel does for one GPU; masked rows get
// 0 everywhere. kl_dir 0 (JSD) writes the LSEs and side outputs only (loss and aux come
// from the second pass).
__global__ void __launch_bounds__(128)
    vp_combine_kernel(const float* __restrict__ st, int n_parts, long long N, const int64_t* __restrict__ labels,
                      long long ignore_index, int kl_dir, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                      float* entropy_s, float* logp_label) {
  pdl_wait();
  pdl_launch_dependents();
  const long long row = blockIdx.x * 128ll + threadIdx.x;
  if (row >= N) return;
  const long long P = (long long)kVpFields * N;   // elements per part
  if (labels[row] == ignore_index) {
    loss_tok[row] = 0.f;
    lse_s[row] = 0.f;
    lse_t[row] = 0.f;
    aux[row] = 0.f;
    if (entropy_s) entropy_s[row] = 0.f;
    if (logp_label) logp_label[row] = 0.f;
    return;
  }
  float ms = kNegBig, mt = kNegBig;
  for (int k = 0; k < n_parts; ++k) {
    ms = fmaxf(ms, st[k * P + row]);
    mt = fmaxf(mt, st[k * P + 2 * N + row]);
  }
  double ls = 0.0, lt = 0.0, a = 0.0, e = 0.0;
  float xl = __int_as_float(0x7fffffff);
  for (int k = 0; k < n_parts; ++k) {
    const float* q = st + k * P;
    const double fs_ = exp2(double(q[row]) - ms), ft_ = exp2(double(q[2 * N + row]) - mt);
    ls += q[N + row] * fs_;
    lt += q[3 * N + row] * ft_;
    if (kl_dir == 1) a += q[4 * N + row] * fs_;
    if (kl_dir == 2) a += q[4 * N + row] * ft_;
    e += (double(q[5 * N + row]) + (double(q[row]) - ms) * q[N + row]) * fs_;
    const float x = q[6 * N + row];
    if (x == x && xl != xl) xl = x;   // first shard that holds the label
  }
  const double L2s = ms + log2(ls), L2t = mt + log2(lt);
  lse_s[row] = float(L2s * 0.69314718055994530942);
  lse_t[row] = float(L2t * 0.69314718055994530942);
  if (entropy_s) entropy_s[row] = float(0.69314718055994530942 * (log2(ls) - e / ls));
  if (logp_label) logp_label[row] = float(0.69314718055994530942 * (double(xl) - L2s));
  float kl = 0.f;
  if (kl_dir == 1) kl = float(0.69314718055994530942 * (a / ls - L2s + L2t));
  if (kl_dir == 2) kl = float(0.69314718055994530942 * (a / lt - L2t + L2s));
  loss_tok[row] = kl;
  aux[row] = kl;
}

// JSD second pass across shards: per valid row, the fixed-order sum of the shards'
// partial sums ([part][2][n_tokens], nats: the divergence and KL(S||M)).
__global__ void __launch_bounds__(128)
    vp_jsd_combine_kernel(const float* __restrict__ parts, int n_parts, long long N,
                          const int64_t* __restrict__ labels, long long ignore_index, float* loss_tok, float* aux) {
  pdl_wait();
  pdl_launch_dependents();
  const long long row = blockIdx.x * 128ll + threadIdx.x;
  if (row >= N) return;
  double js = 0.0, ks = 0.0;
  if (labels[row] != ignore_index)
    for (int k = 0; k < n_parts; ++k) {
      js += parts[k * 2 * N + row];
      ks += parts[k * 2 * N + N + row];
    }
  loss_tok[row] = float(js);
  aux[row] = float(ks);
}

// Masked mean without a workspace: one block counts the valid labels and sums loss_tok
// (masked rows hold 0) in a fixed order, in fp64.
__global__ void __launch_bounds__(1024)
    mean_count_kernel(const float* __restrict__ loss_tok, const int64_t* __restrict__ labels, long long N,
                      long long ignore_index, float* loss_mean, int64_t* n_valid) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ double part[1024];
  __shared__ long long cnt[1024];
  double s = 0.0;
  long long c = 0;
  for (long long i = threadIdx.x; i < N; i += 1024) {
    s += loss_tok[i];
    c += labels[i] != ignore_index;
  }
  part[threadIdx.x] = s;
  cnt[threadIdx.x] = c;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      part[threadIdx.x] += part[threadIdx.x + o];
      cnt[threadIdx.x] += cnt[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *loss_mean = cnt[0] > 0 ? float(part[0] / double(cnt[0])) : 0.f;
    if (n_valid) *n_valid = cnt[0];
  }
}

// ------------------------------------------------------------------ hand-off of hidden rows
// dst row r = src row r for every row whose label is not ignore_index (all rows without
// labels); rows are row_vecs 16-byte vectors. src may be another GPU's memory (a peer or
// IPC mapping): each warp copies one row at a time with four independent 16-byte loads in
// flight per lane, so that many requests cover the link latency; rows are strided over all
// warps of the grid.
__global__ void __launch_bounds__(256)
    handoff_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n_rows,
                        long long row_vecs, const int64_t* __restrict__ labels, long long ignore_index) {
  pdl_wait();
  pdl_launch_dependents();
  const long long warp_id = (blockIdx.x * 256ll + threadIdx.x) >> 5;
  const long long n_warps = (long long)gridDim.x * 8;
  const int lane = threadIdx.x & 31;
  for (long long r = warp_id; r < n_rows; r += n_warps) {
    if (labels && labels[r] == ignore_index) continue;
    const uint4* s = src + r * row_vecs;
    uint4* d = dst + r * row_vecs;
    long long c = lane;
    for (; c + 96 < row_vecs; c += 128) {
      const uint4 a = s[c], b = s[c + 32], e = s[c + 64], f = s[c + 96];
      d[c] = a;
      d[c + 32] = b;
      d[c + 64] = e;
      d[c + 96] = f;
    }
    for (; c < row_vecs; c += 32) d[c] = s[c];
  }
}

// Deterministic masked mean: fixed-order fp64 sum of loss_tok (masked rows hold 0).
__global__ void __launch_bounds__(1024) mean_kernel(const float* __restrict__ loss_tok, int N,
                                                    const Ctrl* __restrict__ ctrl, float* loss_mean) {
  pdl_wait();
  pdl_launch_dependents();
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

// dh_s row r = dh_c[inv[r]] for a valid position (the GEMMs accumulate into the compacted dh_c),
// zeros for a masked one.
__global__ void place_dh_kernel(const float* __restrict__ dhc, int d, float* __restrict__ dh,
                                const int* __restrict__ inv) {
  pdl_wait();
  pdl_launch_dependents();
  const long long r = blockIdx.x;
  const int k = inv[r];
  float4* out = reinterpret_cast<float4*>(dh + r * d);
  if (k < 0) {
    for (int c = threadIdx.x; c < d / 4; c += blockDim.x) out[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    const float4* in = reinterpret_cast<const float4*>(dhc + (long long)k * d);
    for (int c = threadIdx.x; c < d / 4; c += blockDim.x) out[c] = in[c];
  }
}

// ------------------------------------------------------------------ spectral basis selection
// "Nitrobrew tweet analysis", thread item 6/8 and the "SVD-Nitrobrew" row of the evaluation
// table: the teacher code keeps the k right singular vectors of W_t with the largest singular
// values. Given the eigenpairs of G = W_t^T W_t (eigenvalue lambda_i = sigma_i^2, eigenvector i
// in column i of the row-major [d, d] `evecs`, in any order), block i ranks eigenvalue i among
// all d (larger first; equal values by index; NaN last) and, when its rank r is below k, copies
// column i into column r of the basis: V_k (bf16, rounded to nearest even from fp64 once),
// optionally the fp64 copy, and sigma_r = sqrt(max(lambda_i, 0)) (NaN for a NaN eigenvalue).
__device__ __forceinline__ double rank_key(double x) { return isnan(x) ? -INFINITY : x; }

__global__ void __launch_bounds__(256)
    spectral_select_kernel(const double* __restrict__ evals, const double* __restrict__ evecs, int d, int k,
                           __nv_bfloat16* __restrict__ Vk, double* __restrict__ Vk64, double* __restrict__ sigma) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int part[256];
  const int i = blockIdx.x;
  const double li = rank_key(evals[i]);
  int cnt = 0;
  for (int j = threadIdx.x; j < d; j += 256) {
    const double lj = rank_key(evals[j]);
    cnt += (lj > li || (lj == li && j < i)) ? 1 : 0;
  }
  part[threadIdx.x] = cnt;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  const int r = part[0];
  if (r >= k) return;
  if (threadIdx.x == 0) {
    const double l = evals[i];
    sigma[r] = isnan(l) ? l : sqrt(l > 0.0 ? l : 0.0);   // a NaN eigenvalue stays NaN
  }
  for (int a = threadIdx.x; a < d; a += 256) {
    const double v = evecs[(long long)a * d + i];
    Vk[(long long)a * k + r] = __double2bfloat16(v);
    if (Vk64) Vk64[(long long)a * k + r] = v;
  }
}

// Test hook: wait on an mbarrier that nothing arrives at, with the given limit, by polling or
// with the sleeping tests the pipeline kernels use.
__global__ void wait_timeout_kernel(int* status, unsigned long long limit_ns, int sleeping) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl w{status, limit_ns};
    if (sleeping) mbar_wait<true>(&bar, 0, w);
    else mbar_wait<false>(&bar, 0, w);
  }
}

}  // namespace nbkl
