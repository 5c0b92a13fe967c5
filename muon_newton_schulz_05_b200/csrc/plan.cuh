// Internal plan structures shared by the host API and the kernels.
//
// Working layout. Every matrix keeps the layout of its momentum, R x C
// row-major, padded with zeros to Rp x Cp (multiples of 256). A wide matrix
// (R <= C) is iterated as X (r = R): A = X X^T, X <- aX + BX. A tall matrix
// (R > C) is iterated as Y = X^T in the same storage: A = Y^T Y (r = C),
// Y <- aY + Y B (B symmetric). Nothing is ever transposed in memory; the GEMMs
// read the operands K-major or MN-major instead. Zero padding is exact: the
// padded rows and columns of X, A and B stay exactly zero through the
// iteration, because the polynomial is odd.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "muon_b200.h"
#include "check.cuh"
#include "update_math.cuh"

namespace muon {

constexpr int kPad = 256;          // padding granule of R and C
constexpr int kTile = 256;         // GEMM tile (rows and cols) computed by one CTA pair
constexpr int kBM = 128;           // tile rows held by one CTA of the pair
constexpr int kBN = 256;           // tile cols (UMMA N); each CTA loads kBN/2 of B
constexpr int kBK = 64;            // K per pipeline stage (one 128-byte swizzle row)
#ifndef MUON_STAGES
#define MUON_STAGES 4
#endif
#ifndef MUON_EPI_BUFS
#define MUON_EPI_BUFS 3
#endif
constexpr int kStages = MUON_STAGES;  // TMA -> MMA pipeline depth (3 measured slower)
constexpr int kATileBytes = kBM * kBK * 2;
constexpr int kBTileBytes = (kBN / 2) * kBK * 2;
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kEpiWarps = 8;       // two per TMEM lane quadrant
constexpr int kEpiRows = 32;       // epilogue chunk: 32 rows x 32 columns per warp
constexpr int kEpiCols = 32;
constexpr int kEpiHalfBytes = kEpiRows * kEpiCols * 2;      // one bf16 chunk
constexpr int kEpiChunkBytes = 2 * kEpiHalfBytes;           // hi + lo (Apply)
constexpr int kEpiBufs = MUON_EPI_BUFS;                     // chunk buffers per warp
constexpr int kPubSlots = 4;                                // per-CTA publish counters (tiles in flight)
constexpr int kEpiBufBytes = kEpiBufs * kEpiChunkBytes;
constexpr int kGemmSmemBytes = kStages * kStageBytes + kEpiWarps * kEpiBufBytes + 1024 + 512;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;  // warp 0 TMA, warp 1 MMA, then epilogue
constexpr int kChunk = 8192;       // padded elements per block in the momentum pass
constexpr int kMaxMaps = 14;

enum Phase : int { kGram = 0, kPoly = 1, kApply = 2, kReduce = 3 };

// Division by a divisor that is fixed for a launch, as a multiply and a shift
// (division by invariant integers, Granlund and Montgomery): with
// l = ceil(log2 d) and mul = floor(2^32 (2^l - d) / d) + 1,
// n / d = (umulhi(n, mul) + n) >> l for 0 <= n < 2^31.
struct FastDiv {
  uint32_t mul, shift;
};

inline FastDiv make_fastdiv(uint32_t d) {
  if (d == 0) d = 1;  // unused divisors (a phase a bank does not have)
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  const uint64_t mul = ((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1;
  return FastDiv{static_cast<uint32_t>(mul), l};
}

__host__ __device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  const uint32_t u = static_cast<uint32_t>(n);
#ifdef __CUDA_ARCH__
  const uint32_t hi = __umulhi(u, f.mul);
#else
  const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(u) * f.mul) >> 32);
#endif
  return static_cast<int>((hi + u) >> f.shift);
}
constexpr int kRedSub = 4;         // reduce sub-tiles per 256 x 256 tile (32 columns per warp)
constexpr int kMaxSplit = 16;      // K splits of a Gram product

// Tensor-map slots per bank. Operand maps (128-byte swizzle): K-major boxes
// of 128 rows x 64 columns, MN-major boxes of 64 x 64 (the A and B ones read
// a block below the diagonal from its stored transpose). Epilogue maps: 32 x
// 32 chunks, 64-byte swizzle.
enum MapSlot : int {
  kHiK0 = 0, kHiK1 = 1, kHiMN0 = 2, kHiMN1 = 3, kAK = 4, kBK_ = 5,
  kHiE0 = 6, kHiE1 = 7, kLoE = 8, kAE = 9, kAMN = 10, kBE = 11, kBMN = 12,
  kPartE = 13  // fp32 Gram partial tiles, 32 x 32 boxes, 128-byte swizzle
};

struct BankPlan {
  int count, R, C, Rp, Cp, rp, tall;
  int chunks;                   // momentum-pass blocks per matrix
  int tiles_sym;                // upper 256x256 tiles of an rp x rp symmetric product
  int tiles_apply;              // (Rp/256) * (Cp/256)
  int ksplit;                   // K splits of the Gram product (1: none)
  int kc;                       // 64-deep K blocks per split
  int tiles_red;                // reduce sub-tiles (tiles_sym * kRedSub when split)
  FastDiv fd_apply, fd_nbn;     // by tiles_apply, by Cp / 256
  FastDiv fd_gram, fd_ksplit;   // by tiles_sym * ksplit, by ksplit
  FastDiv fd_red, fd_sym;       // by tiles_red, by tiles_sym
  __nv_bfloat16* hi[2];         // iterate, high bf16 part (ping-pong)
  __nv_bfloat16* lo;            // iterate, low bf16 part (in place)
  __nv_bfloat16* A;             // Gram matrix, count x rp x rp; upper 256-blocks only
  __nv_bfloat16* B;             // b A + c A^2, count x rp x rp; upper 256-blocks only
  float* partial;               // count x chunks sums of squares
  float* scale;                 // count: 1 / (||U||_F + eps)
  int* counters;                // count x 4: finished tile parts of Gram, Poly, Apply, Reduce
  float* part;                  // fp32 Gram partials [count][tiles_sym][ksplit][256][256]
};

// Parameter write of one bank (the update pass).
struct UpdBank {
  void* param;          // param (or O output in kUpdWriteO)
  int param_dtype;
  const float* mom_slow;
  float* ema;
  float step_scale;     // lr * max(1, R/C)^(1/2)
};

// ---------------------------------------------------------------- GEMM chain
// One persistent launch runs every Newton-Schulz step of every matrix. Tiles
// are listed step by step, phase by phase (Gram, Reduce, Poly, Apply), bank by
// bank, matrix by matrix; CTA pairs take them round-robin. A tile waits on
// per-matrix counters for the phase it reads. When all eight epilogue warps
// of a CTA have stored their part of an MMA tile (each confirms it after its
// next tile's chunks, or at once when that tile would wait), the last of them
// adds 1 to the tile's phase counter (kTileParts per tile); a Reduce sub-tile
// is published by every epilogue warp of both CTAs (kRedParts). Banks whose
// Gram K is much longer than the matrix is wide split that product along K:
// the split tiles store fp32 partials and Reduce sub-tiles sum them into A.
constexpr int kTileParts = 2;                // MMA tiles: one part per CTA of the pair
constexpr int kRedParts = 2 * kEpiWarps;     // Reduce sub-tiles: one per epilogue warp of both CTAs

struct NsGemmParams {
  CUtensorMap maps[MUON_MAX_BANKS][kMaxMaps];
  BankPlan bank[MUON_MAX_BANKS];
  int gram_begin[MUON_MAX_BANKS + 1];   // prefix sums of count * tiles_sym * ksplit
  int red_begin[MUON_MAX_BANKS + 1];    // prefix sums of count * tiles_red
  int sym_begin[MUON_MAX_BANKS + 1];    // prefix sums of count * tiles_sym
  int apply_begin[MUON_MAX_BANKS + 1];  // prefix sums of count * tiles_apply
  int nbanks;
  int ns_steps;
  FastDiv fd_step;                      // by the tiles of one Newton-Schulz step
  int keep_lo;                          // last step also stores lo (full-precision O)
  float coef[3 * MUON_MAX_NS_STEPS];    // (a, b, c) per step
  int* status;                          // device status word
  unsigned long long wait_limit_ns;
  int fault;                            // test hook (muon_set_debug)
};

__host__ __device__ __forceinline__ int tiles_per_step(const NsGemmParams& p) {
  return p.gram_begin[p.nbanks] + p.red_begin[p.nbanks] + p.sym_begin[p.nbanks] +
         p.apply_begin[p.nbanks];
}

// ---------------------------------------------------------- momentum + norm
struct MomBank {
  const void* grad;
  float* mom;
  float* mom_slow;
  int grad_dtype;
};

enum MomMode : int { kMomMuon = 0, kMomAnvil = 1, kMomNone = 2 };

struct MomParams {
  BankPlan bank[MUON_MAX_BANKS];
  MomBank io[MUON_MAX_BANKS];
  int block_begin[MUON_MAX_BANKS + 1];
  int nbanks;
  int mode;           // MomMode
  float mu;           // Muon mu, or ANVIL beta_fast
  float mu_slow;      // ANVIL beta_slow
  int nesterov;
  int sgd;            // Muon SGD-form momentum (M <- mu M + G)
  float eps;
  int mat_begin[MUON_MAX_BANKS + 1];
  int* status;        // device status word (bounds checks of the debug build)
};

// --------------------------------------------------------------- update pass

struct UpdParams {
  BankPlan bank[MUON_MAX_BANKS];
  UpdBank io[MUON_MAX_BANKS];
  int block_begin[MUON_MAX_BANKS + 1];   // first block of each bank (the momentum pass's grid)
  int nbanks;
  int mode;
  int final_buf;        // hi buffer holding the last iterate
  int use_lo;           // O = hi + lo (else the bf16 hi alone)
  float lr_wd;          // lr * weight_decay
  float ema_beta;
  int* status;          // device status word (bounds checks of the debug build)
};

// Launchers (defined in the .cu files).
cudaError_t launch_momentum_norm(const MomParams& p, int total_blocks, int total_mats,
                                 cudaStream_t s);
cudaError_t launch_ns_gemm(const NsGemmParams& p, int max_pairs, cudaStream_t s);  // whole chain
cudaError_t launch_update(const UpdParams& p, int total_blocks, cudaStream_t s);
cudaError_t launch_ema(float* ema, const void* param, int param_dtype, long long n, float beta,
                       int num_sms, cudaStream_t s);
cudaError_t launch_blend(const void* theta, int theta_dtype, const float* ema, void* out,
                         int out_dtype, long long n, float w_final, int num_sms, cudaStream_t s);
cudaError_t ns_gemm_prepare(int* max_pairs);  // one-time attributes; co-resident CTA pairs

}  // namespace muon
