// Backward GEMMs of one vocabulary chunk on tcgen05 CTA pairs, as one persistent grouped launch.
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
// A pair of CTAs computes a 256 x 256 output tile (cta_group::2): each CTA stages its 128 rows
// of A and 128 of the 256 columns of B, and holds its 128 output rows (one 256-column fp32
// accumulator, double-buffered in TMEM). Wide launches use 256 x 512 tiles instead: both TMEM
// buffers hold one tile, each stage carries A and two B halves, and the epilogue reads the tile
// as two 256-column halves. Same warp roles and barriers as the sweep; warps 4-11 write one
// output row half (128 columns) per thread.
#pragma once

#include "common.cuh"
#include "sweep.cuh"

namespace nbkl {

struct TileInfo {
  int prob, m0, n0, nkb, M;
};

__device__ __forceinline__ int prob_M(const GemmProb& q, int nv) { return q.m_dyn ? nv : q.M; }
__device__ __forceinline__ int prob_K(const GemmProb& q, int nv) {
  // rows n_valid .. (last 256-row tile) of the compacted operands are zeros: K stops at the K
  // block that holds the last valid row
  return q.k_dyn ? ((nv + kBlockK - 1) / kBlockK) * kBlockK : q.K;
}
__device__ __forceinline__ int prob_tiles(const GemmProb& q, int nv, int tile_n) {
  return ((prob_M(q, nv) + kPairM - 1) / kPairM) * ((q.N + tile_n - 1) / tile_n);
}

__device__ __forceinline__ TileInfo tile_info(const GemmArgs& p, int nv, int tile) {
  TileInfo ti;
  const int tile_n = p.wide ? kWideN : kBlockN;
  int pr = 0;
  int t0 = prob_tiles(p.prob[0], nv, tile_n);
  if (p.nprob > 1 && tile >= t0) {
    pr = 1;
    tile -= t0;
  }
  const GemmProb& q = p.prob[pr];
  const int n_tiles = (q.N + tile_n - 1) / tile_n;
  ti.prob = pr;
  ti.m0 = (tile / n_tiles) * kPairM;
  ti.n0 = (tile % n_tiles) * tile_n;
  ti.nkb = (prob_K(q, nv) + kBlockK - 1) / kBlockK;
  ti.M = prob_M(q, nv);
  return ti;
}

__device__ __forceinline__ int total_tiles(const GemmArgs& p, int nv) {
  const int tile_n = p.wide ? kWideN : kBlockN;
  int t = prob_tiles(p.prob[0], nv, tile_n);
  if (p.nprob > 1) t += prob_tiles(p.prob[1], nv, tile_n);
  return t;
}

// Shared-memory addresses of stage `st`'s operands: narrow tiles use kStages x (A, B) of 32 KB;
// wide tiles use the same 192 KB as kWideStages x (A, B half 0, B half 1).
__device__ __forceinline__ uint32_t stage_a(const SweepSmem& s, int wide, int st) {
  return wide ? smem_addr(s.a + st * kWideStageBytes) : stage_a_addr(s, st);
}
__device__ __forceinline__ uint32_t stage_b(const SweepSmem& s, int wide, int st, int half) {
  return wide ? smem_addr(s.a + st * kWideStageBytes + kATileBytes + half * kBTileBytes) : stage_b_addr(s, st);
}

// K-major operand: one (rows x 64) box. MN-major operand: (rows / 64) boxes of 64 x 64
// (64 MN columns each) stacked 8 KB apart. Completed bytes count on the leader's barrier.
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* map, uint32_t bar, int mn_major,
                                             int mn0, int kcoord, int rows) {
  if (!mn_major) {
    tma_load_2d_pair(dst, map, bar, kcoord, mn0);
  } else {
    for (int i = 0; i < rows / 64; ++i) tma_load_2d_pair(dst + i * 8192, map, bar, mn0 + 64 * i, kcoord);
  }
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr, int mn_major, int j) {
  // K-major: 8-row groups 1024 B apart, K step of 16 elements = 32 B inside the swizzle row.
  // MN-major: 64-wide MN atoms 8 KB apart (LBO), 8-row K groups 1024 B apart (SBO),
  // K step of 16 rows = 2048 B.
  return mn_major ? make_sdesc(saddr + j * 2048, 8192, 1024) : make_sdesc(saddr + j * 32, 16, 1024);
}

__device__ __forceinline__ void gemm_producer(const GemmMaps& maps, const GemmArgs& p, int nv, const SweepSmem& s,
                                              const WaitCtl& w, uint32_t rank) {
  int stage = 0;
  uint32_t phase = 0;
  uint32_t pend_stage[kStages];
  uint32_t pend_par[kStages];
  int n_issued = 0;
  bool ok = true;
  const int nt = total_tiles(p, nv);
  const int n_stages = p.wide ? kWideStages : kStages;
  for (int it = 0; ok; ++it) {
    int tile;
    if (rank == 0) {
      tile = next_work(p.sched, it);
      if (tile >= nt) tile = -1;
      if (!ring_put<kGemmSleepProducer>(s, it, tile, w)) { ok = false; break; }
    } else if (!ring_get<kGemmSleepProducer>(s, it, tile, w, false)) {
      ok = false;
      break;
    }
    if (tile < 0) break;
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    const int am0 = ti.m0 + int(rank) * kBlockM, bn0 = ti.n0 + int(rank) * kHalfB;
    for (int kb = 0; kb < ti.nkb; ++kb) {
      if (!mbar_wait_cl<kGemmSleepProducer>(&s.empty[stage], phase ^ 1u, w)) { ok = false; break; }
      const uint32_t bar = smem_addr(&s.full[stage]);
      if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], p.wide ? kWidePairStageBytes : kPairStageBytes);
      const int kc = kb * kBlockK;
      load_operand(stage_a(s, p.wide, stage), &maps.a[ti.prob], bar, q.a_mn, am0, q.a_koff + kc, kBlockM);
      load_operand(stage_b(s, p.wide, stage, 0), &maps.b[ti.prob], bar, q.b_mn, bn0, q.b_koff + kc, kHalfB);
      if (p.wide)   // the second 256-column half of the tile: this CTA's 128 of its B rows
        load_operand(stage_b(s, 1, stage, 1), &maps.b[ti.prob], bar, q.b_mn, bn0 + kBlockN, q.b_koff + kc,
                     kHalfB);
      pend_stage[n_issued % n_stages] = stage;
      pend_par[n_issued % n_stages] = phase;
      ++n_issued;
      if (++stage == n_stages) { stage = 0; phase ^= 1u; }
    }
  }
  if (!ok && rank == 0) drain_loads(s, pend_stage, pend_par, n_issued, n_stages);
}

__device__ __forceinline__ void gemm_mma(const GemmArgs& p, int nv, const SweepSmem& s, uint32_t tmem_base,
                                         const WaitCtl& w) {
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool ok = true;
  for (int it = 0; ok; ++it) {
    int tile;
    if (!ring_get<kGemmSleepMma>(s, it, tile, w, false)) { ok = false; break; }
    if (tile < 0) break;
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    const uint32_t idesc = make_idesc(kPairM, kBlockN, q.a_mn, q.b_mn);
    if (p.wide) {
      // both accumulators hold this tile: columns [n0, n0 + 256) in buffer 0, the next 256 in 1
      if (!mbar_wait_cl<kGemmSleepMma>(&s.tempty[0], acc_phase ^ 1u, w) ||
          !mbar_wait_cl<kGemmSleepMma>(&s.tempty[1], acc_phase ^ 1u, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kb = 0; kb < ti.nkb; ++kb) {
        if (!mbar_wait<kGemmSleepMma>(&s.full[stage], phase, w)) { ok = false; break; }
        const uint32_t sa = stage_a(s, 1, stage);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t sb = stage_b(s, 1, stage, h);
#pragma unroll
          for (int j = 0; j < kBlockK / 16; ++j)
            umma_bf16_pair(tmem_base + h * kBlockN, operand_desc(sa, q.a_mn, j), operand_desc(sb, q.b_mn, j),
                           idesc, (kb > 0 || j > 0) ? 1u : 0u);
          // the first half is complete one half-step early: its epilogue starts meanwhile
          if (h == 0 && kb == ti.nkb - 1) umma_commit_pair_both(smem_addr(&s.tfull[0]));
        }
        umma_commit_pair_both(smem_addr(&s.empty[stage]));
        if (++stage == kWideStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (ti.nkb == 0) umma_commit_pair_both(smem_addr(&s.tfull[0]));
      umma_commit_pair_both(smem_addr(&s.tfull[1]));
      acc_phase ^= 1u;
      continue;
    }
    if (!mbar_wait_cl<kGemmSleepMma>(&s.tempty[acc], acc_phase ^ 1u, w)) { ok = false; break; }
    tc_fence_after();
    const uint32_t d = tmem_base + acc * kBlockN;
    for (int kb = 0; kb < ti.nkb; ++kb) {
      // TMA bytes are ordered by the barrier's transaction count: no tcgen05 fence here
      if (!mbar_wait<kGemmSleepMma>(&s.full[stage], phase, w)) { ok = false; break; }
      const uint32_t sa = stage_a(s, 0, stage);
      const uint32_t sb = stage_b(s, 0, stage, 0);
#pragma unroll
      for (int j = 0; j < kBlockK / 16; ++j) {
        umma_bf16_pair(d, operand_desc(sa, q.a_mn, j), operand_desc(sb, q.b_mn, j), idesc,
                       (kb > 0 || j > 0) ? 1u : 0u);
      }
      umma_commit_pair_both(smem_addr(&s.empty[stage]));
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    if (!ok) break;
    umma_commit_pair_both(smem_addr(&s.tfull[acc]));
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1u;
  }
  if (!ok) drain_mma(s);
}

// Each epilogue warp owns 32 output rows x 128 columns of the pair tile; it moves them in
// 32 x 32 fp32 chunks: TMEM -> registers -> its staging buffer (128-byte swizzle: 16-byte
// piece c of row r sits at piece c ^ (r & 7)) -> one TMA store (or TMA add) per chunk.
// A bf16 output is rounded to nearest even and staged as 64-byte rows (64-byte swizzle:
// piece c of row r at c ^ ((r >> 1) & 3)).
__device__ __forceinline__ void gemm_epilogue(const GemmMaps& maps, const GemmArgs& p, int nv, const SweepSmem& s,
                                              uint32_t tmem_base, const WaitCtl& w) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qq = warp & 3;
  const int half = (warp - kEpiWarp0) >> 2;
  const uint32_t rank = cluster_rank();
  const uint32_t lane_addr = uint32_t(qq * 32) << 16;
  uint8_t* stage = s.out + (warp - kEpiWarp0) * kStageOutBytes;
  uint8_t* stage_row = stage + lane * 128;
  uint8_t* stage_row16 = stage + lane * 64;
  bool staged = false;
  int acc = 0;
  uint32_t acc_phase = 0;
  for (int it = 0;; ++it) {
    int tile;
    if (!ring_get<kGemmSleepEpi>(s, it, tile, w, true)) return;
    if (tile < 0) break;
    const TileInfo ti = tile_info(p, nv, tile);
    const GemmProb& q = p.prob[ti.prob];
    const int row0 = ti.m0 + int(rank) * kBlockM + qq * 32;   // first of the warp's 32 rows
    // a wide tile is read as two 256-column tiles, from accumulator buffers 0 and 1 in turn
#pragma unroll 1
    for (int sub = 0; sub < (p.wide ? 2 : 1); ++sub) {
    const int n0 = ti.n0 + sub * kBlockN;
    if (!mbar_wait_cl<kGemmSleepEpi>(&s.tfull[acc], acc_phase, w)) return;
    tc_fence_after();
    const uint32_t base = tmem_base + lane_addr + acc * kBlockN + half * kHalfN;
#pragma unroll 1
    for (int ch = 0; ch < kHalfN / 32; ++ch) {
      float v[32];
      tmem_ld32(base + ch * 32, v);
      tmem_wait_ld();
      if (ch == kHalfN / 32 - 1) release_accumulator(&s.tempty[acc]);
      if (ti.nkb == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      const int c0 = n0 + half * kHalfN + ch * 32;
      if (c0 >= q.N || row0 >= ti.M) continue;
      if (staged && lane == 0) bulk_wait_read();
      __syncwarp();
      if (q.out_bf16) {
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
          packed[j] = *reinterpret_cast<uint32_t*>(&h2);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(stage_row16 + ((c ^ ((lane >> 1) & 3)) * 16)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(stage_row + ((c ^ (lane & 7)) * 16)) =
              make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (q.accumulate) tma_reduce_add_2d(&maps.out[ti.prob], smem_addr(stage), c0, q.out_row0 + row0);
        else tma_store_2d(&maps.out[ti.prob], smem_addr(stage), c0, q.out_row0 + row0);
        bulk_commit();
      }
      staged = true;
    }
    acc ^= 1;
    if (acc == 0) acc_phase ^= 1u;
    }
  }
  if (lane == 0) bulk_wait_all();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const SweepSmem s = carve_smem(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.nprob; ++i) {
      tma_prefetch_map(&maps.a[i]);
      tma_prefetch_map(&maps.b[i]);
      tma_prefetch_map(&maps.out[i]);
    }
  }
  const uint32_t tmem_base = pair_prologue(s);
  pdl_wait();
  pdl_launch_dependents();
  const int nv = *p.n_valid;
  const WaitCtl w{p.status, p.wait_limit_ns};
  if (warp < kEpiWarp0) {
    regs_shrink<kRegsCtl>();
    if (warp == 0 && lane == 0) gemm_producer(maps, p, nv, s, w, rank);
    if (warp == 1 && lane == 0 && rank == 0) gemm_mma(p, nv, s, tmem_base, w);
  } else {
    regs_grow<kRegsEpi>();
    gemm_epilogue(maps, p, nv, s, tmem_base, w);
  }
  pair_epilogue(s, tmem_base, w);
}

}  // namespace nbkl
