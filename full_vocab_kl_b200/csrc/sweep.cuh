// Vocabulary sweep: both block GEMMs on tcgen05 with a fused per-token epilogue.
//
// "Nitrobrew tweet analysis", section "Nitrobrew 的两个动作": for each vocabulary
// block, z_s = h_s W_s[v0:v1]^T and z_t = h_t W_t[v0:v1]^T are formed, the online
// softmax / log-sum-exp accumulators and the KL terms are updated, and the block is
// discarded. Here one block is a 256-token x 256-column tile computed by a pair of CTAs
// (cta_group::2): each CTA stages 128 token rows of h and 128 vocabulary rows of W per K step
// and holds its 128 rows of both fp32 accumulators.
//
// Tensor memory holds both accumulators of a tile (2 x 256 columns = all 512), so it cannot be
// double-buffered. Instead the model with the larger K ("first") is multiplied first and
// committed on its own barrier; the epilogue copies the first accumulator into registers while
// the second model's MMAs run and releases it, so the next tile's first-model MMAs can start as
// soon as the tile ends, while the epilogue streams the second accumulator (released after its
// last read, normally long before the next tile's first-model phase ends).
//
// Warp roles (384 threads per CTA, one CTA per SM, persistent over work units):
//   warp 0     TMA producer (both CTAs): 128 x 64 h tile + 128 x 64 W tile per stage, 7 stages
//              (6 in the gradient sweep, whose epilogue stages its output in the 7th)
//   warp 1     MMA issuer (leader CTA only): 4 x tcgen05.mma 256x256x16 per K block; TMEM owner
//   warps 2-3  idle (warpgroup 0 hands its registers to the epilogue: 56 vs 224 per thread)
//   warps 4-11 epilogue: two warps per TMEM lane quarter, each thread one token row and one
//              128-column half of the tile, base-2 online math in registers
//
// Barriers: the leader's full[] barrier counts the TMA bytes of both CTAs; the MMA completion
// is multicast to the empty[] / tfull[] barriers of both CTAs; the epilogue warps of both CTAs
// arrive on the leader's tempty[]. Work ids come from the leader's TMA thread through a ring
// mirrored into the peer CTA.
//
// A work unit is (256-row token tile, run of vocabulary tiles: `tiles_per_unit` of them for the
// first `n_big` vocabulary units, one for the rest); each thread writes its row's partial state
// once per unit (split = 2 * vocabulary unit + column half).
#pragma once

#include "common.cuh"

namespace nbkl {

struct SweepSmem {
  uint8_t* a;           // operand stages: kMaxStages x (A 16 KB, B 16 KB); wide GEMM tiles 4 x 48 KB
  uint8_t* out;         // kEpiWarps x 4 KB TMA-store staging (over the 7th stage; 6-stage kernels only)
  uint64_t* full;       // kMaxStages (leader: TMA bytes of both CTAs)
  uint64_t* empty;      // kMaxStages (both: MMA commit)
  uint64_t* tfull;      // sweep: [1] first model, [0] whole tile complete; GEMM: one per stage
  uint64_t* tempty;     // leader: accumulator released by all 16 epilogue warps of the pair
  uint64_t* drain;      // 1
  uint64_t* ring_full;  // kRing: a work id was written to ring_slot (both CTAs)
  uint64_t* ring_empty; // kRing: leader: every consumer of the pair has read it
  int* ring_slot;       // kRing
  uint32_t* tmem_slot;
};

__device__ __forceinline__ SweepSmem carve_smem(uint8_t* raw) {
  SweepSmem s;
  uint8_t* base = align1024(raw);
  s.a = base;
  s.out = base + kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kMaxStages * kStageBytes);
  s.full = bars;
  s.empty = bars + kMaxStages;
  s.tfull = bars + 2 * kMaxStages;
  s.tempty = bars + 2 * kMaxStages + 2;
  s.drain = bars + 2 * kMaxStages + 4;
  s.ring_full = bars + 2 * kMaxStages + 5;
  s.ring_empty = s.ring_full + kRing;
  s.ring_slot = reinterpret_cast<int*>(s.ring_empty + kRing);
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.ring_slot + kRing);
  return s;
}

// Operand tiles of narrow stage `st`.
__device__ __forceinline__ uint32_t stage_a_addr(const SweepSmem& s, int st) {
  return smem_addr(s.a + st * kStageBytes);
}
__device__ __forceinline__ uint32_t stage_b_addr(const SweepSmem& s, int st) {
  return smem_addr(s.a + st * kStageBytes + kATileBytes);
}

__device__ __forceinline__ void init_barriers(const SweepSmem& s) {
  for (int i = 0; i < kMaxStages; ++i) {
    mbar_init(&s.full[i], 1);
    mbar_init(&s.empty[i], 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(&s.tfull[i], 1);
    mbar_init(&s.tempty[i], 2 * kEpiWarps);
  }
  mbar_init(s.drain, 1);
  for (int i = 0; i < kRing; ++i) {
    mbar_init(&s.ring_full[i], 1);
    mbar_init(&s.ring_empty[i], kRingConsumers);
  }
  fence_mbar_init();
}

// Common prologue of the pair kernels: barriers, TMEM (512 columns in each CTA), cluster sync.
__device__ __forceinline__ uint32_t pair_prologue(const SweepSmem& s) {
  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) init_barriers(s);
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(s.tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any cross-CTA arrive or TMA byte count
  tc_fence_after();
  return *s.tmem_slot;
}

__device__ __forceinline__ void pair_epilogue(const SweepSmem& s, uint32_t tmem_base, const WaitCtl& w) {
  const int warp = threadIdx.x / 32;
  tc_fence_before();
  __syncthreads();
  if (*reinterpret_cast<volatile int*>(w.status) != 0) {
    // after a failure, give copies the peer may still have in flight time to land
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) {
    }
  }
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

struct UnitGrid {
  int n_valid, n_tt, n_vt, n_vu, n_units;
};

// Vocabulary units: the first n_big units are runs of tiles_per_unit tiles, the rest single tiles
// (n_big * tiles_per_unit <= n_vt), so the last work items of a launch are short.
__device__ __forceinline__ UnitGrid unit_grid(const SweepArgs& p) {
  UnitGrid g;
  g.n_valid = *p.n_valid;
  g.n_tt = (g.n_valid + kPairM - 1) / kPairM;
  g.n_vt = (p.v_end - p.v_begin + kBlockN - 1) / kBlockN;
  g.n_vu = p.n_big + (g.n_vt - p.n_big * p.tiles_per_unit);
  g.n_units = g.n_tt * g.n_vu;
  return g;
}

// Work order: token tiles in groups of tt_group; within a group, vocabulary-unit major (the
// group's token tiles of one vocabulary unit are consecutive work items, so the pairs working at
// the same time share the unembedding tiles), and a group's units all come before the next
// group's (so the compacted rows re-read for every vocabulary tile stay few enough for L2).
__device__ __forceinline__ void decode_unit(const SweepArgs& p, const UnitGrid& g, int u, int& vu, int& tt) {
  const int G = p.tt_group;
  const int n_full = g.n_tt / G;
  const int per_group = G * g.n_vu;
  if (u < n_full * per_group) {
    const int grp = u / per_group, r = u % per_group;
    vu = r / G;
    tt = grp * G + r % G;
  } else {
    const int rem = g.n_tt - n_full * G, r = u - n_full * per_group;
    vu = r / rem;
    tt = n_full * G + r % rem;
  }
}

// First and one-past-last vocabulary tile of vocabulary unit vu.
__device__ __forceinline__ int unit_t0(const SweepArgs& p, int vu) {
  return vu < p.n_big ? vu * p.tiles_per_unit : p.n_big * p.tiles_per_unit + (vu - p.n_big);
}
__device__ __forceinline__ int unit_t1(const SweepArgs& p, int vu) {
  return vu < p.n_big ? (vu + 1) * p.tiles_per_unit : unit_t0(p, vu) + 1;
}

// ------------------------------------------------------------------ work distribution
// The leader's TMA thread takes the next work id (from a global counter when `sched` is set,
// so that pairs which start late, or share the GPU with another kernel, simply take fewer
// items; else a static stride over pairs), writes it into the ring of both CTAs and arrives on
// both ring_full[] barriers. The leader's MMA thread, the peer's TMA thread and the epilogue
// warps of both CTAs read it and arrive on the leader's ring_empty[]. -1 ends the sequence.
__device__ __forceinline__ int next_work(int* sched, int it) {
  const int pair = int(blockIdx.x) >> 1, n_pairs = int(gridDim.x) >> 1;
  return sched ? atomicAdd(sched, 1) : pair + it * n_pairs;
}

template <bool kSleep>
__device__ __forceinline__ bool ring_put(const SweepSmem& s, int it, int id, const WaitCtl& w) {
  const int k = it % kRing;
  if (!mbar_wait_cl<kSleep>(&s.ring_empty[k], ((it / kRing) & 1) ^ 1, w)) return false;
  s.ring_slot[k] = id;
  st_remote_u32(cluster_addr(smem_addr(&s.ring_slot[k]), 1), uint32_t(id));
  mbar_arrive(&s.ring_full[k]);
  mbar_arrive_remote(cluster_addr(smem_addr(&s.ring_full[k]), 1));
  return true;
}

// `warp_wide`: every lane waits and reads, lane 0 arrives once for the warp.
template <bool kSleep>
__device__ __forceinline__ bool ring_get(const SweepSmem& s, int it, int& id, const WaitCtl& w, bool warp_wide) {
  const int k = it % kRing;
  if (!mbar_wait_cl<kSleep>(&s.ring_full[k], (it / kRing) & 1, w)) return false;
  id = *reinterpret_cast<volatile int*>(&s.ring_slot[k]);
  if (warp_wide) __syncwarp();
  if (!warp_wide || (threadIdx.x % 32) == 0)
    mbar_arrive_remote(cluster_addr(smem_addr(&s.ring_empty[k]), 0));
  return true;
}

// Bounded wait for the copies a failed producer may still have in flight (leader: its full[]
// barriers count the bytes of both CTAs).
// `pend_*` hold the stage and parity of the last `n_stages` loads, at index (load number) % n_stages.
__device__ __forceinline__ void drain_loads(const SweepSmem& s, const uint32_t* pend_stage,
                                            const uint32_t* pend_par, int n_issued, int n_stages) {
  const int n = min(n_issued, n_stages);
  for (int i = 0; i < n; ++i) {
    const int j = (n_issued - 1 - i) % n_stages;
    const uint32_t a = smem_addr(&s.full[pend_stage[j]]);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_test(a, pend_par[j]) && global_timer_ns() - t0 < 100000000ull) {
    }
  }
}

// Bounded wait until every pair MMA the leader issued has completed.
__device__ __forceinline__ void drain_mma(const SweepSmem& s) {
  umma_commit_pair_local(smem_addr(s.drain));
  const uint32_t a = smem_addr(s.drain);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_test(a, 0) && global_timer_ns() - t0 < 100000000ull) {
  }
}

// Epilogue warp's release of a TMEM accumulator: after its own tcgen05.ld completed, lane 0
// arrives on the leader's barrier.
__device__ __forceinline__ void release_accumulator(uint64_t* bar) {
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x % 32) == 0) mbar_arrive_remote(cluster_addr(smem_addr(bar), 0));
}

// ------------------------------------------------------------------ producer (both CTAs)
template <int NST>
__device__ __forceinline__ void sweep_producer(const SweepMaps& maps, const SweepArgs& p, const UnitGrid& g,
                                               const SweepSmem& s, const WaitCtl& w, uint32_t rank) {
  int stage = 0;
  uint32_t phase = 0;
  uint32_t pend_stage[NST], pend_par[NST];
  int n_issued = 0;
  // first model = teacher when teacher_first
  const CUtensorMap* a1 = p.teacher_first ? &maps.a_t : &maps.a_s;
  const CUtensorMap* b1 = p.teacher_first ? &maps.b_t : &maps.b_s;
  const CUtensorMap* a2 = p.teacher_first ? &maps.a_s : &maps.a_t;
  const CUtensorMap* b2 = p.teacher_first ? &maps.b_s : &maps.b_t;
  const int nk1 = p.teacher_first ? p.nkb_t : p.nkb_s, nk2 = p.teacher_first ? p.nkb_s : p.nkb_t;
  const int bm1 = p.teacher_first ? p.bmod_t : p.bmod_s, bm2 = p.teacher_first ? p.bmod_s : p.bmod_t;
  bool ok = true;
  for (int it = 0; ok; ++it) {
    int u;
    if (rank == 0) {
      u = next_work(p.sched, it);
      if (u >= g.n_units) u = -1;
      if (!ring_put<kSweepSleepProducer>(s, it, u, w)) { ok = false; break; }
    } else if (!ring_get<kSweepSleepProducer>(s, it, u, w, false)) {
      ok = false;
      break;
    }
    if (u < 0) break;
    int vu, tt;
    decode_unit(p, g, u, vu, tt);
    const int row0 = tt * kPairM + int(rank) * kBlockM;
    const int t_end = unit_t1(p, vu);
    for (int t = unit_t0(p, vu); t < t_end && ok; ++t) {
      const int v0 = p.v_begin + t * kBlockN + int(rank) * kHalfB;
      for (int kb = 0; kb < nk1 + nk2; ++kb) {
        if (!mbar_wait_cl<kSweepSleepProducer>(&s.empty[stage], phase ^ 1u, w)) { ok = false; break; }
        const bool one = kb < nk1;
        const int k = one ? kb : kb - nk1;
        const int kbb = k % (one ? bm1 : bm2);
        const uint32_t bar = smem_addr(&s.full[stage]);
        if (rank == 0) mbar_arrive_expect_tx(&s.full[stage], kPairStageBytes);
        tma_load_2d_pair(stage_a_addr(s, stage), one ? a1 : a2, bar, k * kBlockK, row0);
        tma_load_2d_pair(stage_b_addr(s, stage), one ? b1 : b2, bar, kbb * kBlockK, v0);
        pend_stage[n_issued % NST] = stage;
        pend_par[n_issued % NST] = phase;
        ++n_issued;
        if (++stage == NST) { stage = 0; phase ^= 1u; }
      }
    }
  }
  if (!ok && rank == 0) drain_loads(s, pend_stage, pend_par, n_issued, NST);
}

// ------------------------------------------------------------------ MMA issuer (leader)
template <int NST>
__device__ __forceinline__ void sweep_mma(const SweepArgs& p, const UnitGrid& g, const SweepSmem& s,
                                          uint32_t tmem_base, const WaitCtl& w) {
  int stage = 0;
  uint32_t phase = 0;
  uint32_t lt = 0;  // tiles processed by this pair
  const int nk1 = p.teacher_first ? p.nkb_t : p.nkb_s, nk2 = p.teacher_first ? p.nkb_s : p.nkb_t;
  bool ok = true;
  for (int it = 0; ok; ++it) {
    int u;
    if (!ring_get<kSweepSleepMma>(s, it, u, w, false)) { ok = false; break; }
    if (u < 0) break;
    int vu, tt;
    decode_unit(p, g, u, vu, tt);
    const int t_end = unit_t1(p, vu);
    for (int t = unit_t0(p, vu); t < t_end && ok; ++t, ++lt) {
      for (int kb = 0; kb < nk1 + nk2; ++kb) {
        const bool one = kb < nk1;
        const int k = one ? kb : kb - nk1;
        if (k == 0) {
          // the accumulator of this model must have been read by both CTAs' epilogues
          if (!mbar_wait_cl<kSweepSleepMma>(&s.tempty[one ? 0 : 1], (lt & 1u) ^ 1u, w)) { ok = false; break; }
          tc_fence_after();
        }
        // TMA bytes are ordered by the barrier's transaction count: no tcgen05 fence here
        if (!mbar_wait<kSweepSleepMma>(&s.full[stage], phase, w)) { ok = false; break; }
        const uint32_t d = tmem_base + (one ? 0 : kBlockN);
        const uint32_t sa = stage_a_addr(s, stage);
        const uint32_t sb = stage_b_addr(s, stage);
#pragma unroll
        for (int j = 0; j < kBlockK / 16; ++j) {
          umma_bf16_pair(d, make_sdesc(sa + j * 32, 16, 1024), make_sdesc(sb + j * 32, 16, 1024), kIdescKK,
                         (k > 0 || j > 0) ? 1u : 0u);
        }
        umma_commit_pair_both(smem_addr(&s.empty[stage]));
        if (++stage == NST) { stage = 0; phase ^= 1u; }
        // first accumulator complete: the epilogues copy it out while the second model runs
        if (kb == nk1 - 1) umma_commit_pair_both(smem_addr(&s.tfull[1]));
      }
      if (!ok) break;
      umma_commit_pair_both(smem_addr(&s.tfull[0]));
    }
  }
  if (!ok) drain_mma(s);
}

// ------------------------------------------------------------------ epilogue math
// Online base-2 state of one token row: running maxima m, rescaled sums l = sum 2^(x - m),
// and a = sum 2^(x_p - m_p) (x_p - x_q) for the model p the KL takes its expectation under.
// With side outputs, e = sum 2^(x_s - m_s) (x_s - m_s): every term is <= 0, so the student
// entropy ln 2 * (log2 l_s - e / l_s) is formed without cancellation.
struct RowState {
  float ms, ls, mt, lt, a, e;
};

// One 32-column chunk of a row: zs / zt hold the raw logits z. The maxima are taken on z (the
// scale log2(e) / tau is positive) and every exponent is formed as fma(z, scale, -m), so the
// scaled logits are never stored; the KL numerator sums 2^(x - m) (z_s - z_t) in raw units and
// is scaled once per chunk. Column pairs go through the packed f32x2 forms.
template <int MODE, bool MASKED, bool SIDE>
__device__ __forceinline__ void chunk_state(float (&zs)[32], float (&zt)[32], int n_ok, float scale, RowState& r,
                                            int lab_off, float* lab_dst) {
  if (MASKED) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j >= n_ok) { zs[j] = kNegBig; zt[j] = kNegBig; }
  }
  float cs = zs[0], ct = zt[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) {
    cs = fmaxf(cs, zs[j]);
    ct = fmaxf(ct, zt[j]);
  }
  const float ns = fmaxf(r.ms, cs * scale), nt = fmaxf(r.mt, ct * scale);
  const float rs = ex2(r.ms - ns), rt = ex2(r.mt - nt);
  // re-centre e on the new maximum: sum 2^(x - ns) (x - ns) = rs (e + (ms - ns) l)
  if (SIDE) r.e = rs * fmaf(r.ms - ns, r.ls, r.e);
  r.ls *= rs;
  r.lt *= rt;
  if (MODE == kStateS) r.a *= rs;
  if (MODE == kStateT) r.a *= rt;
  r.ms = ns;
  r.mt = nt;
  const f2 sc = pk2(scale, scale), mns = pk2(-ns, -ns), mnt = pk2(-nt, -nt), m1 = pk2(-1.f, -1.f);
  f2 ls = pk2(0.f, 0.f), lt = ls, a = ls, e = ls;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const f2 z_s = pk2(zs[j], zs[j + 1]), z_t = pk2(zt[j], zt[j + 1]);
    f2 ds = fma2(z_s, sc, mns), dt = fma2(z_t, sc, mnt);   // x - m
    float d0, d1, t0, t1;
    upk2(ds, d0, d1);
    upk2(dt, t0, t1);
    if (MASKED) {
      // columns past the vocabulary contribute exactly 0 whatever the running maximum (when a
      // thread's first chunk is all masked, fma(z, scale, -m) would leave the product's
      // rounding error of a huge value here instead of 0)
      if (j >= n_ok) d0 = t0 = kNegBig;
      if (j + 1 >= n_ok) d1 = t1 = kNegBig;
      ds = pk2(d0, d1);
    }
    const f2 es = pk2(ex2(d0), ex2(d1)), et = pk2(ex2(t0), ex2(t1));
    ls = add2(ls, es);
    lt = add2(lt, et);
    if (SIDE) e = fma2(es, ds, e);
    if (MODE == kStateS) a = fma2(es, fma2(z_t, m1, z_s), a);
    if (MODE == kStateT) a = fma2(et, fma2(z_s, m1, z_t), a);
  }
  r.ls += sum2(ls);
  r.lt += sum2(lt);
  if (MODE == kStateS || MODE == kStateT) r.a = fmaf(sum2(a), scale, r.a);
  if (SIDE) {
    r.e += sum2(e);
    // the one thread whose chunk holds the row's label keeps that logit (a rare branch)
    if (unsigned(lab_off) < 32u) {
      float z = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) z = (j == lab_off) ? zs[j] : z;
      *lab_dst = z * scale;
    }
  }
}

struct RowConst {
  float l2s, l2t, aux;
  float beta, omb;
};

// log2 of the mixture M = (1 - beta) S + beta T from S and T themselves, floored at 2^-126:
// where both have underflowed every term that uses it is below 2^-126 anyway.
__device__ __forceinline__ f2 log2_mix2(f2 S, f2 T, f2 omb, f2 bb) {
  float m0, m1;
  upk2(fma2(bb, T, mul2(omb, S)), m0, m1);
  return pk2(lg2(fmaxf(m0, 0x1p-126f)), lg2(fmaxf(m1, 0x1p-126f)));
}

// JSD pass: js += beta sum T (y_t - y_m) + (1 - beta) sum S (y_s - y_m), ks += sum S (y_s - y_m)
// (base 2, converted to nats by the finalisation), column pairs in packed form.
template <bool MASKED>
__device__ __forceinline__ void chunk_jsd(const float (&zs)[32], const float (&zt)[32], int n_ok, float scale,
                                          const RowConst& c, float& js, float& ks) {
  const f2 sc = pk2(scale, scale), ms = pk2(-c.l2s, -c.l2s), mt = pk2(-c.l2t, -c.l2t), m1 = pk2(-1.f, -1.f);
  const f2 omb = pk2(c.omb, c.omb), bb = pk2(c.beta, c.beta);
  f2 k_acc = pk2(0.f, 0.f), j_acc = k_acc;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const f2 ys = fma2(pk2(zs[j], zs[j + 1]), sc, ms), yt = fma2(pk2(zt[j], zt[j + 1]), sc, mt);
    float s0, s1, t0, t1;
    upk2(ys, s0, s1);
    upk2(yt, t0, t1);
    float S0 = ex2(s0), S1 = ex2(s1), T0 = ex2(t0), T1 = ex2(t1);
    if (MASKED && j >= n_ok) S0 = T0 = 0.f;
    if (MASKED && j + 1 >= n_ok) S1 = T1 = 0.f;
    const f2 S = pk2(S0, S1), T = pk2(T0, T1);
    const f2 ym = log2_mix2(S, T, omb, bb);
    k_acc = fma2(S, fma2(ym, m1, ys), k_acc);
    j_acc = fma2(T, fma2(ym, m1, yt), j_acc);
  }
  // JSD = beta * KL(T||M) + (1 - beta) * KL(S||M); the S term is the K accumulator
  const float k = sum2(k_acc);
  js += fmaf(c.beta, sum2(j_acc), c.omb * k);
  ks += k;
}

// Gradient of one 32-column chunk of a row, packed to bf16 and written into the warp's
// staging buffer (32 rows x 64 bytes, 64-byte swizzle: 16-byte piece c of row r sits at piece
// c ^ ((r >> 1) & 3)), from where one TMA store per warp writes the 32 x 32 block.
template <int MODE, bool MASKED>
__device__ __forceinline__ void chunk_grad(const float (&zs)[32], const float (&zt)[32], int n_ok, float scale,
                                           const RowConst& c, float gs, uint8_t* stage_row, int r) {
  uint32_t packed[16];
  // the two KL directions in packed pairs: y = fma(z, scale, -L2) are the base-2 log-probabilities
  const f2 sc = pk2(scale, scale), ms = pk2(-c.l2s, -c.l2s), mt = pk2(-c.l2t, -c.l2t), m1 = pk2(-1.f, -1.f);
  const f2 ln2 = pk2(kLn2, kLn2), maux = pk2(-c.aux, -c.aux), g2 = pk2(gs, gs);
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float g0, g1;
    if (MODE == kGradFkl || MODE == kGradRkl) {
      const f2 ys = fma2(pk2(zs[j], zs[j + 1]), sc, ms), yt = fma2(pk2(zt[j], zt[j + 1]), sc, mt);
      float s0, s1, t0, t1;
      upk2(ys, s0, s1);
      upk2(yt, t0, t1);
      const f2 S = pk2(ex2(s0), ex2(s1));
      f2 g;
      if (MODE == kGradFkl) {
        g = fma2(pk2(ex2(t0), ex2(t1)), m1, S);                    // S - T
      } else {
        g = mul2(S, fma2(ln2, fma2(yt, m1, ys), maux));            // S (ln S - ln T - KL)
      }
      upk2(mul2(g, g2), g0, g1);
    } else {
      // (1 - beta) S (ln S - ln M - K)
      const f2 ys = fma2(pk2(zs[j], zs[j + 1]), sc, ms), yt = fma2(pk2(zt[j], zt[j + 1]), sc, mt);
      float s0, s1, t0, t1;
      upk2(ys, s0, s1);
      upk2(yt, t0, t1);
      const f2 S = pk2(ex2(s0), ex2(s1)), T = pk2(ex2(t0), ex2(t1));
      const f2 ym = log2_mix2(S, T, pk2(c.omb, c.omb), pk2(c.beta, c.beta));
      const f2 g = mul2(mul2(S, pk2(c.omb, c.omb)), fma2(ln2, fma2(ym, m1, ys), maux));
      upk2(mul2(g, g2), g0, g1);
    }
    if (MASKED && j >= n_ok) g0 = 0.f;
    if (MASKED && j + 1 >= n_ok) g1 = 0.f;
    __nv_bfloat162 h = __floats2bfloat162_rn(g0, g1);
    packed[j / 2] = *reinterpret_cast<uint32_t*>(&h);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(stage_row + ((q ^ ((r >> 1) & 3)) * 16)) =
        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

template <int MODE>
__device__ __forceinline__ void process_chunk(float (&zs)[32], float (&zt)[32], int n_ok, const SweepArgs& p,
                                              const RowConst& c, float gs, RowState& r, float& js, float& ks,
                                              uint8_t* gstage, int lane, int lab_off, float* lab_dst) {
  const bool masked = n_ok < 32;
  if (MODE <= kStateT) {
    if (p.side) {
      if (masked) chunk_state<MODE, true, true>(zs, zt, n_ok, p.scale, r, lab_off, lab_dst);
      else chunk_state<MODE, false, true>(zs, zt, n_ok, p.scale, r, lab_off, lab_dst);
    } else {
      if (masked) chunk_state<MODE, true, false>(zs, zt, n_ok, p.scale, r, -1, nullptr);
      else chunk_state<MODE, false, false>(zs, zt, n_ok, p.scale, r, -1, nullptr);
    }
  } else if (MODE == kJsd) {
    if (masked) chunk_jsd<true>(zs, zt, n_ok, p.scale, c, js, ks);
    else chunk_jsd<false>(zs, zt, n_ok, p.scale, c, js, ks);
  } else {
    if (masked) chunk_grad<MODE, true>(zs, zt, n_ok, p.scale, c, gs, gstage, lane);
    else chunk_grad<MODE, false>(zs, zt, n_ok, p.scale, c, gs, gstage, lane);
  }
}

// ------------------------------------------------------------------ epilogue
template <int MODE>
__device__ __forceinline__ void sweep_epilogue(const SweepMaps& maps, const SweepArgs& p, const UnitGrid& g,
                                               const SweepSmem& s, uint32_t tmem_base, const WaitCtl& w) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int q = warp & 3;                      // TMEM lane quarter this warp may access
  const int half = (warp - kEpiWarp0) >> 2;    // column half of the tile
  const int row_in_tile = q * 32 + lane;
  const uint32_t lane_addr = uint32_t(q * 32) << 16;
  const uint32_t rank = cluster_rank();
  uint8_t* stage = s.out + (warp - kEpiWarp0) * kStageOutBytes;
  uint8_t* stage_row = stage + lane * 64;
  bool staged = false;                                           // a TMA store may still read it
  const uint32_t col1 = tmem_base + lane_addr + half * kHalfN;   // first model
  const uint32_t col2 = col1 + kBlockN;                          // second model
  uint32_t lt = 0;
  RowConst c;
  c.beta = p.beta;
  c.omb = 1.0f - p.beta;
  const float gscale = (MODE >= kGradFkl) ? *p.gscale : 0.f;

  for (int it = 0;; ++it) {
    int u;
    if (!ring_get<kSweepSleepEpi>(s, it, u, w, true)) return;
    if (u < 0) break;
    int vu, tt;
    decode_unit(p, g, u, vu, tt);
    const int row = tt * kPairM + int(rank) * kBlockM + row_in_tile;
    const bool row_ok = row < g.n_valid;
    if (MODE >= kJsd) {
      c.l2s = p.row_l2s[row];
      c.l2t = p.row_l2t[row];
      c.aux = p.row_aux[row];
    }
    const float gs = row_ok ? gscale : 0.f;
    // label column of this row (side outputs of the state passes), -1 when none
    const int lab = (MODE <= kStateT && p.side && row_ok) ? p.row_label[row] : -1;
    float* const lab_dst = (MODE <= kStateT && p.side) ? p.label_x + row : nullptr;
    RowState r{kNegBig, 0.f, kNegBig, 0.f, 0.f, 0.f};
    float js = 0.f, ks = 0.f;
    const int t_end = unit_t1(p, vu);
    for (int t = unit_t0(p, vu); t < t_end; ++t, ++lt) {
      const int v0 = p.v_begin + t * kBlockN + half * kHalfN;
      if (!mbar_wait_cl<kSweepSleepEpi>(&s.tfull[1], lt & 1u, w)) return;   // first model complete
      tc_fence_after();
      float F[4][32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(col1 + ch * 32, F[ch]);
      tmem_wait_ld();
      release_accumulator(&s.tempty[0]);
      if (!mbar_wait_cl<kSweepSleepEpi>(&s.tfull[0], lt & 1u, w)) return;   // second model complete
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float C[32];
        tmem_ld32(col2 + ch * 32, C);
        tmem_wait_ld();
        if (ch == 3) release_accumulator(&s.tempty[1]);
        const int c0 = v0 + ch * 32;
        const int n_ok = p.V - c0;            // columns of this chunk inside the vocabulary
        if (MODE >= kGradFkl) {
          if (staged && lane == 0) bulk_wait_read();
          __syncwarp();
        }
        const int lab_off = lab < 0 ? -1 : lab - c0;
        if (p.teacher_first) process_chunk<MODE>(C, F[ch], n_ok, p, c, gs, r, js, ks, stage_row, lane, lab_off, lab_dst);
        else process_chunk<MODE>(F[ch], C, n_ok, p, c, gs, r, js, ks, stage_row, lane, lab_off, lab_dst);
        if (MODE >= kGradFkl) {
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&maps.g_out, smem_addr(stage), c0 - p.v_begin, row - lane);
            bulk_commit();
          }
          staged = true;
        }
      }
    }
    const long long off = (long long)(2 * vu + half) * p.ld + row;
    if (MODE <= kStateT) {
      p.out[off] = r.ms;
      p.out[p.field_stride + off] = r.ls;
      p.out[2 * p.field_stride + off] = r.mt;
      p.out[3 * p.field_stride + off] = r.lt;
      p.out[4 * p.field_stride + off] = r.a;
      if (p.side) p.out[5 * p.field_stride + off] = r.e;
    } else if (MODE == kJsd) {
      p.out[off] = js;
      p.out[p.field_stride + off] = ks;
    }
  }
  if (MODE >= kGradFkl && lane == 0) bulk_wait_all();
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sweep_kernel(const __grid_constant__ SweepMaps maps, const SweepArgs p) {
  extern __shared__ uint8_t smem_raw[];
  const SweepSmem s = carve_smem(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&maps.a_s);
    tma_prefetch_map(&maps.b_s);
    tma_prefetch_map(&maps.a_t);
    tma_prefetch_map(&maps.b_t);
    if (MODE >= kGradFkl) tma_prefetch_map(&maps.g_out);
  }
  const uint32_t tmem_base = pair_prologue(s);
  pdl_wait();
  pdl_launch_dependents();
  const UnitGrid g = unit_grid(p);
  const WaitCtl w{p.status, p.wait_limit_ns};

  // the gradient sweep stages its output tiles, the state and JSD sweeps take a 7th operand stage
  constexpr int NST = MODE >= kGradFkl ? kStages : kMaxStages;
  if (warp < kEpiWarp0) {
    regs_shrink<kRegsCtl>();
    if (warp == 0 && lane == 0) sweep_producer<NST>(maps, p, g, s, w, rank);
    if (warp == 1 && lane == 0 && rank == 0) sweep_mma<NST>(p, g, s, tmem_base, w);
  } else {
    regs_grow<kRegsEpi>();
    sweep_epilogue<MODE>(maps, p, g, s, tmem_base, w);
  }
  pair_epilogue(s, tmem_base, w);
}

}  // namespace nbkl
