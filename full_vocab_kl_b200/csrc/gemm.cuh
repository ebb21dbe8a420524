// Backward GEMMs of one vocabulary chunk on tcgen05, as one persistent grouped launch.
//
// "Nitrobrew tweet analysis", section "仓库实现": the gradient flows only to the student
// hidden state and the student unembedding, and the logit blocks are recomputed in the
// backward pass rather than kept. With G = dL/dz_s for the chunk's columns (bf16, staged
// by the gradient sweep), the two products are
//   dh_s[rows]   (+)= G          @ W_s[chunk]      (M = tokens, N = d_s, K = chunk columns)
//   dW_s[chunk]  (+)= G^T        @ h_s[valid rows] (M = chunk columns, N = d_s, K = tokens)
// G^T, W_s[chunk] (as K x N) and h_s (as K x N) are read MN-major straight from their
// row-major buffers through 64 x 64 TMA boxes, so nothing is transposed in memory.
//
// Same warp roles as the sweep: warp 0 TMA, warp 1 MMA (one 128 x 256 fp32 accumulator,
// double-buffered in TMEM), warps 4-11 write one output row half (128 columns) per thread.
#pragma once

#include "common.cuh"
#include "sweep.cuh"

namespace nbkl {

struct TileInfo {
  int prob, m0, n0, nkb, M;
};

__device__ __forceinline__ int prob_M(const GemmProb& q, int nv) { return q.m_dyn ? nv : q.M; }
__device__ __forceinline__ int prob_K(const GemmProb& q, int nv) {
  return q.k_dyn ? ((nv + kBlockM - 1) / kBlockM) * kBlockM : q.K;
}
__device__ __forceinline__ int prob_tiles(const GemmProb& q, int nv) {
  return ((prob_M(q, nv) + kBlockM - 1) / kBlockM) * ((q.N + kBlockN - 1) / kBlockN);
}

__device__ __forceinline__ TileInfo tile_info(const GemmArgs& p, int nv, int tile) {
  TileInfo ti;
  int pr = 0;
  int t0 = prob_tiles(p.prob[0], nv);
  if (p.nprob > 1 && tile >= t0) {
    pr = 1;
    tile -= t0;
  }
  const GemmProb& q = p.prob[pr];
  const int n_tiles = (q.N + kBlockN - 1) / kBlockN;
  ti.prob = pr;
  ti.m0 = (tile / n_tiles) * kBlockM;
  ti.n0 = (tile % n_tiles) * kBlockN;
  ti.nkb = (prob_K(q, nv) + kBlockK - 1) / kBlockK;
  ti.M = prob_M(q, nv);
  return ti;
}

__device__ __forceinline__ int total_tiles(const GemmArgs& p, int nv) {
  int t = prob_tiles(p.prob[0], nv);
  if (p.nprob > 1) t += prob_tiles(p.prob[1], nv);
  return t;
}

// K-major operand: one (rows x 64) box. MN-major operand: (rows / 64) boxes of 64 x 64
// (64 MN columns each) stacked 8 KB apart.
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* map, uint32_t bar, int mn_major,
                                             int mn0, int kcoord, int rows) {
  if (!mn_major) {
    tma_load_2d(dst, map, bar, kcoord, mn0);
  } else {
    for (int i = 0; i < rows / 64; ++i) tma_load_2d(dst + i * 8192, map, bar, mn0 + 64 * i, kcoord);
  }
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr, int mn_major, int j) {
  // K-major: 8-row groups 1024 B apart, K step of 16 elements = 32 B inside the swizzle row.
  // MN-major: 64-wide MN atoms 8 KB apart (LBO), 8-row K groups 1024 B apart (SBO),
  // K step of 16 rows = 2048 B.
  return mn_major ? make_sdesc(saddr + j * 2048, 8192, 1024) : make_sdesc(saddr + j * 32, 16, 1024);
}

__device__ __forceinline__ void gemm_producer(const GemmMaps& maps, const GemmArgs& p, int nv, const SweepSmem& s,
                                              const WaitCtl& w) {
  int stage = 0;
  uint32_t phase = 0;
  uint32_t pend_stage[kStages];
  uint32_t pend_par[kStages];
  int n_issued = 0;
  bool ok = true;
  const int nt = total_tiles(p, nv);
  for (int tile = blockIdx.x; tile < nt && ok; tile += gridDim.x) {
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    for (int kb = 0; kb < ti.nkb; ++kb) {
      if (!mbar_wait(&s.empty[stage], phase ^ 1u, w)) { ok = false; break; }
      const uint32_t bar = smem_addr(&s.full[stage]);
      mbar_arrive_expect_tx(&s.full[stage], kStageBytes);
      load_operand(smem_addr(s.a + stage * kATileBytes), &maps.a[ti.prob], bar, q.a_mn, ti.m0,
                   q.a_koff + kb * kBlockK, kBlockM);
      load_operand(smem_addr(s.b + stage * kBTileBytes), &maps.b[ti.prob], bar, q.b_mn, ti.n0,
                   q.b_koff + kb * kBlockK, kBlockN);
      pend_stage[n_issued % kStages] = stage;
      pend_par[n_issued % kStages] = phase;
      ++n_issued;
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
  }
  if (!ok) drain_loads(s, pend_stage, pend_par, n_issued);
}

__device__ __forceinline__ void gemm_mma(const GemmArgs& p, int nv, const SweepSmem& s, uint32_t tmem_base,
                                         const WaitCtl& w) {
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool ok = true;
  const int nt = total_tiles(p, nv);
  for (int tile = blockIdx.x; tile < nt && ok; tile += gridDim.x) {
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    const uint32_t idesc = make_idesc(kBlockM, kBlockN, q.a_mn, q.b_mn);
    if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, w)) { ok = false; break; }
    tc_fence_after();
    const uint32_t d = tmem_base + acc * kBlockN;
    for (int kb = 0; kb < ti.nkb; ++kb) {
      if (!mbar_wait(&s.full[stage], phase, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_addr(s.a + stage * kATileBytes);
      const uint32_t sb = smem_addr(s.b + stage * kBTileBytes);
#pragma unroll
      for (int j = 0; j < kBlockK / 16; ++j) {
        umma_bf16(d, operand_desc(sa, q.a_mn, j), operand_desc(sb, q.b_mn, j), idesc, (kb > 0 || j > 0) ? 1u : 0u);
      }
      umma_commit(smem_addr(&s.empty[stage]));
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    if (!ok) break;
    umma_commit(smem_addr(&s.tfull[acc]));
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1u;
  }
  if (!ok) drain_mma(s);
}

__device__ __forceinline__ void gemm_epilogue(const GemmArgs& p, int nv, const SweepSmem& s, uint32_t tmem_base,
                                              const WaitCtl& w) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qq = warp & 3;
  const int half = (warp - kEpiWarp0) >> 2;
  const uint32_t lane_addr = uint32_t(qq * 32) << 16;
  int acc = 0;
  uint32_t acc_phase = 0;
  const int nt = total_tiles(p, nv);
  for (int tile = blockIdx.x; tile < nt; tile += gridDim.x) {
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    const int m = ti.m0 + qq * 32 + lane;
    const bool row_ok = m < ti.M;
    float* orow = nullptr;
    if (row_ok) {
      const long long r = q.row_map ? (long long)q.row_map[m] : (long long)(q.row_off + m);
      orow = q.out + r * q.ldo;
    }
    if (!mbar_wait(&s.tfull[acc], acc_phase, w)) return;
    tc_fence_after();
    const uint32_t base = tmem_base + lane_addr + acc * kBlockN + half * kHalfN;
#pragma unroll 1
    for (int ch = 0; ch < kHalfN / 32; ++ch) {
      float v[32];
      tmem_ld32(base + ch * 32, v);
      tmem_wait_ld();
      if (ch == kHalfN / 32 - 1) {
        tc_fence_before();
        mbar_arrive(&s.tempty[acc]);
      }
      if (ti.nkb == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      const int c0 = ti.n0 + half * kHalfN + ch * 32;
      if (!row_ok || c0 >= q.N) continue;
      float* dst = orow + c0;
      if (c0 + 32 <= q.N) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 o = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          if (q.accumulate) {
            const float4 old = d4[j];
            o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
          }
          d4[j] = o;
        }
      } else {
        for (int j = 0; j < q.N - c0; ++j) dst[j] = q.accumulate ? dst[j] + v[j] : v[j];
      }
    }
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1u;
  }
}

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const SweepSmem s = carve_smem(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) init_barriers(s);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.nprob; ++i) {
      tma_prefetch_map(&maps.a[i]);
      tma_prefetch_map(&maps.b[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(s.tmem_slot), 2 * kBlockN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;
  const int nv = *p.n_valid;
  const WaitCtl w{p.status, p.wait_limit_ns};
  if (warp < kEpiWarp0) {
    regs_shrink<kRegsCtl>();
    if (warp == 0 && lane == 0) gemm_producer(maps, p, nv, s, w);
    if (warp == 1 && lane == 0) gemm_mma(p, nv, s, tmem_base, w);
  } else {
    regs_grow<kRegsEpi>();
    gemm_epilogue(p, nv, s, tmem_base, w);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kBlockN);
  }
}

}  // namespace nbkl
