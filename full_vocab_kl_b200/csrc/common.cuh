// Tile geometry, kernel argument blocks and small helpers shared by the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace nbkl {

// A pair of CTAs (a cluster of 2, one per SM) owns a 256-token x 256-column output tile: the
// tcgen05 MMA is 256 x 256 x 16 with cta_group::2. Each CTA stages its own 128 rows of A and
// 128 of the 256 rows of B (so an SM loads half of B per FLOP), and keeps its 128 rows of
// the fp32 accumulators in its tensor memory. K advances 64 bf16 (one 128-byte swizzle row)
// per pipeline stage. (A single-CTA 128 x 128 MMA keeps the tensor pipe as busy as a 128 x 256
// one for half the work, and a single-CTA 128 x 256 GEMM reached only ~63% of cuBLAS here.)
constexpr int kBlockM = 128;                           // rows per CTA
constexpr int kPairM = 2 * kBlockM;                    // rows per pair (MMA M)
constexpr int kBlockN = 256;                           // MMA N
constexpr int kHalfB = kBlockN / 2;                    // B rows staged per CTA
constexpr int kBlockK = 64;
// Pipeline stages: 6 for the kernels that also stage output tiles for TMA stores (gradient
// sweep, GEMM), 7 for the state and JSD sweeps, whose 7th stage takes the output staging area.
constexpr int kStages = 6;
constexpr int kMaxStages = 7;
constexpr int kATileBytes = kBlockM * kBlockK * 2;     // 16 KB
constexpr int kBTileBytes = kHalfB * kBlockK * 2;      // 16 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes; // 32 KB per CTA: A tile, then B tile
constexpr int kPairStageBytes = 2 * kStageBytes;       // bytes the leader's full barrier expects
constexpr int kEpiWarps = 8;                           // two warps per TMEM lane quarter
constexpr int kEpiWarp0 = 4;                           // epilogue = warpgroups 1 and 2
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 128 + kEpiThreads;            // warpgroup 0: TMA warp, MMA warp, 2 idle
// Register split: warpgroup 0 gives registers back, the epilogue warpgroups take them.
// 128 * kRegsCtl + 256 * kRegsEpi must not exceed 384 * (registers at launch = 168).
constexpr int kRegsLaunch = 168;
constexpr int kRegsCtl = 56;
constexpr int kRegsEpi = 224;

// Which roles wait with sleeping barrier tests (descheduled until the phase completes) rather
// than by polling. The MMA issuer's wait for a stage's operands is on the critical path, and a
// polling wait could see the landed operands up to a microsecond late; every role sleeps.
constexpr bool kSweepSleepEpi = true, kSweepSleepProducer = true, kSweepSleepMma = true;
constexpr bool kGemmSleepEpi = true, kGemmSleepProducer = true, kGemmSleepMma = true;
static_assert(128 * kRegsCtl + kEpiThreads * kRegsEpi <= kThreads * kRegsLaunch, "register split");
constexpr int kHalfN = kBlockN / 2;                    // columns per epilogue thread per tile
// Per epilogue warp, one 4 KB staging buffer for TMA stores (32 rows x 128 bytes, 128-byte
// swizzle: fp32 32 x 32 chunks of the GEMM output, bf16 32 x 32 chunks of the gradient).
constexpr int kStageOutBytes = 4096;
static_assert(kStages * kStageBytes + kEpiWarps * kStageOutBytes <= kMaxStages * kStageBytes,
              "output staging fits in the 7th stage");
constexpr int kSmemBytes = kMaxStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

constexpr int kRing = 4;                               // work ids in flight inside a pair
constexpr int kRingConsumers = 2 * (1 + 8);            // per CTA: MMA or TMA thread + 8 epilogue warps

constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kNegBig = -1.0e30f;  // finite "minus infinity" for masked columns

// Idesc of the sweep's 256 x 256 K-major x K-major pair products.
constexpr uint32_t kIdescKK = make_idesc(kPairM, kBlockN, 0, 0);

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------ vocabulary sweep
enum SweepMode : int {
  kStateNone = 0,   // pass 1 of the JSD: online (max, sum) of both models
  kStateS = 1,      // reverse KL: + E_S[u_s - u_t] accumulator
  kStateT = 2,      // forward KL: + E_T[u_t - u_s] accumulator
  kJsd = 3,         // pass 2 of the JSD with the final LSEs
  kGradFkl = 4,     // backward, beta = 0
  kGradRkl = 5,     // backward, beta = 1
  kGradJsd = 6,     // backward, beta in (0, 1)
};

struct SweepMaps {
  CUtensorMap a_s, b_s, a_t, b_t;   // compacted h_s, W_s, compacted h_t, W_t
  CUtensorMap g_out;                // backward: gradient chunk, bf16, 32 x 32 boxes, 64-byte swizzle
};

struct SweepArgs {
  int teacher_first;      // MMA order / epilogue order: the model with the larger K goes first
  int V;                  // vocabulary size
  int v_begin, v_end;     // vocabulary columns covered by this launch
  int nkb_s, nkb_t;       // K blocks of the A operands (student, teacher)
  int bmod_s, bmod_t;     // B block of A block kb is kb % bmod (fp32 hi/lo split reuses W)
  int tiles_per_unit;     // vocabulary tiles per work unit of the first n_big units (one split of the
  int n_big;              // LSE state each); every later unit is a single tile (a short tail of work)
  float scale;            // log2(e) / tau: base-2 tempered logits x = z * scale
  float beta;
  float* out;             // state [6][split][ld] or JSD partial sums [2][split][ld]; split =
                          // 2 * unit + column half
  long long field_stride; // elements between fields of `out`
  int ld;                 // rows per split in `out`
  const float* row_l2s;   // per compacted row: base-2 LSE of the student (pass 2, backward)
  const float* row_l2t;
  const float* row_aux;   // per compacted row: per-token KL (beta = 1) or KL(S||M) (JSD)
  int side;               // forward state passes: also the student entropy accumulator and the
                          // tempered logit of each row's label
  const int* row_label;   // per compacted row: label column, or -1 (side outputs)
  float* label_x;         // per compacted row: base-2 tempered student logit at the label
  __nv_bfloat16* G;       // backward: gradient chunk [rows][ldG]
  long long ldG;
  const float* gscale;    // device scalar grad_out / (N_v * tau)
  const int* n_valid;     // device scalar
  int* sched;             // zeroed work counter: CTAs take units in order (null: static stride)
  int* status;
  unsigned long long wait_limit_ns;
  int tt_group;           // token tiles per group of the work order (all vocabulary units of one
                          // group before the next group)
};

// ------------------------------------------------------------------ backward GEMMs
struct GemmMaps {
  CUtensorMap a[2], b[2];
  CUtensorMap out[2];               // fp32 outputs, 32 x 32 boxes, 128-byte swizzle
};

struct GemmProb {
  int a_mn, b_mn;          // operand majorness (1 = MN-major)
  int a_koff, b_koff;      // K coordinate offsets of the operands
  int m_dyn, M;            // m_dyn: M = n_valid (else M)
  int N;
  int k_dyn, K;            // k_dyn: K = round_up(n_valid, 64) (else K)
  int out_row0;            // output-map row of tile row 0
  int accumulate;          // 1: out += acc (TMA reduce-add), 0: out = acc (TMA store)
  int out_bf16;            // 1: out is bf16 (32 x 32 boxes, 64-byte swizzle), stored rounded to nearest even
};

// Wide GEMM tiles: 256 x 512 per CTA pair (two N = 256 accumulators, all of TMEM), 4 stages of
// A 16 KB + B 2 x 16 KB per CTA. Each stage's operand bytes then feed twice the MMA work of
// a 256 x 256 tile's stage with half again as many bytes: 25% fewer shared-memory writes
// per FLOP.
constexpr int kWideN = 2 * kBlockN;                         // 512
constexpr int kWideStages = 4;
constexpr int kWideStageBytes = kATileBytes + 2 * kBTileBytes;   // 48 KB per CTA
constexpr int kWidePairStageBytes = 2 * kWideStageBytes;
static_assert(kWideStages * kWideStageBytes == kStages * kStageBytes, "wide stages reuse the operand area");

struct GemmArgs {
  GemmProb prob[2];
  int nprob;
  int wide;                // 1: every tile is 256 x 512 (kWideN); 0: 256 x 256, double-buffered
  const int* n_valid;
  int* sched;              // zeroed work counter (null: static stride)
  int* status;
  unsigned long long wait_limit_ns;
};

}  // namespace nbkl
