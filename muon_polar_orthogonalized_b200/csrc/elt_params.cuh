// elt_params.cuh -- parameter blocks of the elementwise kernels (momentum,
// Frobenius finalize, update, NorMuon, AdamW), built by the host planner and
// passed by value (__grid_constant__).
#pragma once
#include "common.cuh"

namespace muon {

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
  int item_begin;    // momentum_bulk: first stage item (two chunks) of this matrix
  int sidx;          // index of this matrix's scale in the wave's scale array
  float lr;          // lr * lr_scale (update kernel)
  int pbase;         // MuonEq momentum: index of the first row's partial in `partials`
};

struct EltParams {
  MatRef mats[kMaxMatsPerLaunch];
  int nmats;
  int total_blocks;  // work chunks (one partial sum each); blocks loop over them
  int total_items;   // momentum_bulk: stage items (up to two chunks of one matrix)
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
  unsigned int* status;   // momentum_bulk: status word (a bounded wait ran out)
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
  float rsqrt_bc2;   // 1 / sqrt(1 - beta2^t)
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

// ------------------------------------------------------------- replicate
// Copies of parameter matrices: dst[r][i] <- src[i] for r < nrep, for the
// update paths that do not write the copies themselves.
constexpr int kReplMats = 64;
struct ReplParams {
  const float* src[kReplMats];
  float* dst[kMaxReplicas][kReplMats];
  long long numel[kReplMats];
  int blk_begin[kReplMats];   // first work chunk of matrix i
  int nmats;
  int nrep;
  int total_blocks;
};

// ------------------------------------------------------------ reduce_mean
// dst[i] <- (src[0][i] + src[1][i] + ... + src[n-1][i]) * (1/n), summed in
// fp32 in that order; tensors fp32 or bf16 (one dtype per launch).
constexpr int kMaxSources = 8;
constexpr int kMeanTensors = 64;
struct MeanParams {
  const void* src[kMaxSources][kMeanTensors];
  void* dst[kMeanTensors];
  long long numel[kMeanTensors];
  int blk_begin[kMeanTensors];
  int ntensors;
  int nsrc;
  int total_blocks;
  int bf16;
  float inv_n;
};

}  // namespace muon
