// common.cuh -- parameter blocks shared by the host planner and the kernels.
// Every pointer table travels as a by-value (__grid_constant__) kernel
// parameter, so a step needs no device-side descriptor copies and can be
// captured in a CUDA graph.
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

// Status word bits recorded by device code (OR-ed into workspace word 0).
constexpr uint32_t kDevTimeout = 1u;

// Device-resident schedule state (layout of muon_schedule_state): every
// learning rate is multiplied by lr_mult; AdamW's bias correction uses step.
struct DevSched {
  float lr_mult;
  float reserved;
  long long step;
};

// ------------------------------------------------- elementwise: per matrix
struct MatRef {
  const void* g;     // gradient (or orthogonaliser input), rows x cols, dense
  float* m;          // momentum (nullptr: orthogonaliser mode, m~ = g)
  float* w;          // parameters (update kernel)
  float* out;        // fp32 output (emit kernel)
  void* x;           // workspace X buffer of this matrix (bf16 or fp32), pitch ldx
  int rows, cols, ldx;
  int vec;           // 1: 4-wide vector path is legal for this matrix
  int blk_begin;     // first block of this matrix in the launch
  int sidx;          // index of this matrix's scale in the wave's scale array
  float lr;          // lr * lr_scale (update kernel)
  int pbase;         // MuonEq momentum: index of the first row's partial in `partials`
};

struct EltParams {
  MatRef mats[kMaxMatsPerLaunch];
  int nmats;
  int total_blocks;  // work chunks (one partial sum each); blocks loop over them
  int grid;          // launched blocks (persistent, <= total_blocks)
  int grad_bf16;     // grads of every matrix in this launch are bf16
  int x_f32;         // workspace X is fp32 (debug mode)
  int nesterov;
  float beta;
  float wd;
  int cautious;
  int use_scale;     // update/emit: multiply X by the matrix scale (ns_steps == 0)
  int row_eq;        // MuonEq: momentum kernel row-wise, one partial sum per row
  float* partials;   // momentum kernel: one partial sum of squares per block (or row)
  float* scales;     // per-matrix 1/(||m~||+eps)
  const DevSched* sched;  // nullptr, or the device schedule (lr multiplier)
};

// ------------------------------------------------------------ GEMM problems
enum EpiKind : int { EPI_GRAM = 0, EPI_POLY = 1, EPI_AXPY = 2, EPI_AXPY_UPDATE = 3 };

// One problem = `batch` same-shape matrices laid out at a fixed batch stride.
//   C[i][j] = sum_k Aop(i,k) * Bop(j,k)
//   Aop(i,k) = a[i*lda + k] (K-major) or a[k*lda + i] (MN-major), same for Bop.
struct GemmProblem {
  int M, N, K, batch;
  int a_mn, b_mn;
  int sym;                  // output symmetric: upper tiles computed and mirrored
  int tiles_m, tiles_n, tiles_per_mat, tile_begin;
  // operands (SIMT path reads these directly; the tensor-core path uses tensor maps)
  const void* a; long long a_bs; int a_ld;
  const void* b; long long b_bs; int b_ld;
  // epilogue
  void* out; long long out_bs; int out_ld;
  const void* ein; long long ein_bs; int ein_ld;   // A (poly) or X (axpy)
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
  GemmProblem prob[kMaxProblems];
  float* wptr[kMaxUpdMats];
  int wcols[kMaxUpdMats];   // param row pitch (= cols)
  int nprob;
  int total_tiles;
  const float* scales;
  unsigned int* status;
  float wd;
  int cautious;
  const DevSched* sched;
};

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

// ---------------------------------------------------------------- AdamW
struct AdamTensor {
  float* p;
  const void* g;
  float* m;
  float* v;
  long long numel;
  int blk_begin;
  int vec;
  float decay;       // 1 - lr*wd
  float b1, omb1;    // beta1, 1 - beta1
  float b2, omb2;
  float step_size;   // lr / (1 - beta1^t)
  float sqrt_bc2;    // sqrt(1 - beta2^t)
  float eps;
  float lr, wd;      // base values (device schedule: the scalars above are recomputed)
};

struct AdamParams {
  AdamTensor t[kMaxAdamTensors];
  int ntensors;
  int total_blocks;  // work chunks
  int grid;          // launched blocks (persistent)
  int grad_bf16;
  const DevSched* sched;  // nullptr, or the device schedule (lr multiplier, step)
};

}  // namespace muon
