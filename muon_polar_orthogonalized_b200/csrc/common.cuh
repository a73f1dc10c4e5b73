// common.cuh -- limits, the device schedule state and the GEMM parameter
// blocks shared by the host planner and the Newton-Schulz kernels (the
// elementwise kernels' blocks are in elt_params.cuh).  Every pointer table
// travels as a by-value (__grid_constant__) kernel parameter, so a step needs
// no device-side descriptor copies and can be captured in a CUDA graph.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace muon {

// ------------------------------------------------------------------ limits
constexpr int kMaxMatsPerLaunch = 256;   // elementwise launches (momentum, update, emit)
constexpr int kMaxProblems = 16;         // GEMM launches: (group slice) problems per launch
constexpr int kMaxUpdMats = 256;         // fused-update pointer table
constexpr int kMaxAdamTensors = 128;     // AdamW tensors per launch
constexpr int kWsHeaderBytes = 4096;     // workspace header: status word + reserve
constexpr int kMaxNsSteps = 16;
constexpr int kMaxReplicas = 7;          // copies of W written with the update (the other ranks of a node)

// Status word bits recorded by device code (OR-ed into workspace word 0).
constexpr uint32_t kDevTimeout = 1u;

// Device-resident schedule state (layout of muon_schedule_state): every
// learning rate is multiplied by lr_mult; AdamW's bias correction uses step.
struct DevSched {
  float lr_mult;
  float reserved;
  long long step;
};

// ------------------------------------------------------------ GEMM problems
enum EpiKind : int { EPI_GRAM = 0, EPI_POLY = 1, EPI_AXPY = 2, EPI_AXPY_UPDATE = 3 };

// One problem = `batch` same-shape matrices laid out at a fixed batch stride.
//   C[i][j] = sum_k Aop(i,k) * Bop(j,k)
//   Aop(i,k) = a[i*lda + k] (K-major) or a[k*lda + i] (MN-major), same for Bop.
// Symmetric m x m matrices (A, B') are stored by the tensor-core path in
// "upper" form: element (i, j) is written only where j/256 >= i/256 (the
// 256x256 blocks on and above the diagonal, diagonal blocks in full).  A
// product that reads such an operand takes a K block that lies left of the
// operand rows' diagonal block from the stored block above the diagonal,
// transposed (an MN-major load of rows k, columns i: the value at (k, i) is
// the one (i, k) would hold).
constexpr int kSymBlock = 256;

struct GemmProblem {
  int M, N, K, batch;
  int a_mn, b_mn;
  int sym;                  // output symmetric: upper tiles computed, upper form stored
  int a_sym, b_sym;         // operand stored in upper form (tensor-core path)
  int tiles_m, tiles_n, tiles_per_mat, tile_begin;
  int col_major;            // tile order of a non-symmetric output: tile rows fastest
                            // (else bands of tile columns, tile columns fastest)
  int chunked;              // tensor-core path: every operand row length is a multiple
                            // of 64, and the tensor maps are chunked 4-D views (one
                            // box per operand per pipeline stage)
  // operands (SIMT path reads these directly; the tensor-core path uses tensor maps)
  const void* a; long long a_bs; int a_ld;
  const void* b; long long b_bs; int b_ld;
  // epilogue
  void* out; long long out_bs; int out_ld;
  const void* ein; long long ein_bs; int ein_ld;   // A (poly) or X (axpy)
  // exact diagonal of B' (tensor-core path): the A*A epilogue writes, per
  // row, r_i = B'_ii / bf16(B'_ii) (fp32); the B'X epilogue multiplies the
  // product's row i (wide) or column i (tall, dsc_col = 1) by r_i, which
  // makes the diagonal term exact
  float* dsc; long long dsc_bs; int dsc_col;
  int scale_mode;           // 0 none, 1: s^2 (first Gram), 2: s (first X update)
  int scale_base;           // index of matrix 0 of this problem in the scale array
  float ca, cb, cc;         // a_k, b_k, c_k
  // fused update
  int w_first;              // index of matrix 0 in the update pointer table
  float lr;                 // lr * lr_scale of this group
};

struct alignas(64) TcGemmParams {
  CUtensorMap tmA[kMaxProblems];
  CUtensorMap tmB[kMaxProblems];
  CUtensorMap tmA2[kMaxProblems];   // MN-major boxes of an upper-form A operand (its K blocks left of the diagonal)
  CUtensorMap tmB2[kMaxProblems];   // likewise for B
  CUtensorMap tmOut[kMaxProblems];  // output rows of Gram and B'X: 32x32 boxes, 64-byte swizzle
  GemmProblem prob[kMaxProblems];
  float* wptr[kMaxUpdMats];
  int wcols[kMaxUpdMats];   // param row pitch (= cols)
  float* rptr[kMaxReplicas][kMaxUpdMats];   // fused update: copies of each W written with it
  int nrep;                 // copies in rptr (0: none)
  int nprob;
  int total_tiles;
  const float* scales;
  unsigned int* status;
  float wd;
  int cautious;
  const DevSched* sched;
};
static_assert(sizeof(TcGemmParams) <= 32764, "kernel parameter limit");

struct SimtGemmParams {
  GemmProblem prob[kMaxProblems];
  float* wptr[kMaxUpdMats];
  int wcols[kMaxUpdMats];
  int nprob;
  int total_tiles;
  const float* scales;
  float wd;
  int cautious;
  const DevSched* sched;
};

}  // namespace muon
