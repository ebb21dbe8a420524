// Tile geometry, kernel argument blocks and small helpers shared by the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace nbkl {

// One CTA owns a 128-token x 256-column output tile (the MMA instruction is 128 x 256 x 16:
// with N = 128 the tensor pipe stays busy for the same time and delivers half the work);
// K advances 64 bf16 (one 128-byte swizzle row) per pipeline stage.
constexpr int kBlockM = 128;
constexpr int kBlockN = 256;
constexpr int kBlockK = 64;
constexpr int kStages = 4;
constexpr int kATileBytes = kBlockM * kBlockK * 2;     // 16 KB
constexpr int kBTileBytes = kBlockN * kBlockK * 2;     // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes; // 48 KB
constexpr int kEpiWarps = 8;                           // two warps per TMEM lane quarter
constexpr int kEpiWarp0 = 4;                           // epilogue = warpgroups 1 and 2
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 128 + kEpiThreads;            // warpgroup 0: TMA warp, MMA warp, 2 idle
// Register split: warpgroup 0 gives registers back, the epilogue warpgroups take them.
// 128 * kRegsCtl + 256 * kRegsEpi must not exceed 384 * (registers at launch = 168).
constexpr int kRegsLaunch = 168;
constexpr int kRegsCtl = 56;
constexpr int kRegsEpi = 224;
static_assert(128 * kRegsCtl + kEpiThreads * kRegsEpi <= kThreads * kRegsLaunch, "register split");
constexpr int kHalfN = kBlockN / 2;                    // columns per epilogue thread per tile
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kNegBig = -1.0e30f;  // finite "minus infinity" for masked columns

// Idesc of the sweep's 128 x 256 K-major x K-major products.
constexpr uint32_t kIdescKK = make_idesc(kBlockM, kBlockN, 0, 0);

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
};

struct SweepArgs {
  int teacher_first;      // MMA order / epilogue order: the model with the larger K goes first
  int V;                  // vocabulary size
  int v_begin, v_end;     // vocabulary columns covered by this launch
  int nkb_s, nkb_t;       // K blocks of the A operands (student, teacher)
  int bmod_s, bmod_t;     // B block of A block kb is kb % bmod (fp32 hi/lo split reuses W)
  int tiles_per_unit;     // vocabulary tiles per work unit (one split of the LSE state)
  float scale;            // log2(e) / tau: base-2 tempered logits x = z * scale
  float beta, lg2_1mb, lg2_b;
  float* out;             // state [5][split][ld] or JSD partial sums [2][split][ld]; split =
                          // 2 * unit + column half
  long long field_stride; // elements between fields of `out`
  int ld;                 // rows per split in `out`
  const float* row_l2s;   // per compacted row: base-2 LSE of the student (pass 2, backward)
  const float* row_l2t;
  const float* row_aux;   // per compacted row: per-token KL (beta = 1) or KL(S||M) (JSD)
  __nv_bfloat16* G;       // backward: gradient chunk [rows][ldG]
  long long ldG;
  const float* gscale;    // device scalar grad_out / (N_v * tau)
  const int* n_valid;     // device scalar
  int* status;
  unsigned long long wait_limit_ns;
};

// ------------------------------------------------------------------ backward GEMMs
struct GemmMaps {
  CUtensorMap a[2], b[2];
};

struct GemmProb {
  int a_mn, b_mn;          // operand majorness (1 = MN-major)
  int a_koff, b_koff;      // K coordinate offsets of the operands
  int m_dyn, M;            // m_dyn: M = n_valid (else M)
  int N;
  int k_dyn, K;            // k_dyn: K = round_up(n_valid, 128) (else K)
  float* out;
  long long ldo;
  const int* row_map;      // output row of tile row m (null: row_off + m)
  int row_off;
  int accumulate;          // 1: out += acc, 0: out = acc
};

struct GemmArgs {
  GemmProb prob[2];
  int nprob;
  const int* n_valid;
  int* status;
  unsigned long long wait_limit_ns;
};

}  // namespace nbkl
