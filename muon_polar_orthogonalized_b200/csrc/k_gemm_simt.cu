// k_gemm_simt.cu -- fp32-operand Newton-Schulz products for the debug mode.
//
// Same three products and epilogues as the tensor-core kernels (Gram,
// B' = a*I + b*A + c*A*A, B'*X, and the fused cautious update), but with fp32 operands and
// fp32 FMA accumulation on the CUDA cores, so the whole iteration can be
// checked to ~1e-6 against the fp64 oracle.  Correctness scaffold, not a fast
// path: 64x64 tiles, 16x16 threads with 4x4 outputs each, full (not
// triangular) outputs.
#include <cuda_runtime.h>

#include "common.cuh"
#include "pdl.cuh"

namespace muon {

constexpr int ST_BM = 64, ST_BN = 64, ST_BK = 16;

__device__ __forceinline__ float op_load(const float* base, int ld, int mn, int idx_mn, int k, int ext_mn, int K) {
  if (idx_mn >= ext_mn || k >= K) return 0.f;
  return mn ? base[static_cast<long long>(k) * ld + idx_mn] : base[static_cast<long long>(idx_mn) * ld + k];
}

__device__ __forceinline__ float cautious_w_f32(float w, float u, float lr, float wd, bool cautious) {
  bool mask = true;
  if (cautious) {
    const bool sdiff = (__float_as_uint(u) ^ __float_as_uint(w)) >> 31;
    mask = !sdiff || u == 0.f || w == 0.f;
  }
  const float t = mask ? fmaf(wd, w, u) : u;
  return fmaf(-lr, t, w);
}

template <int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const __grid_constant__ SimtGemmParams p) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float As[ST_BK][ST_BM + 1];
  __shared__ float Bs[ST_BK][ST_BN + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
    int pi = 0;
    while (pi + 1 < p.nprob && t >= p.prob[pi + 1].tile_begin) ++pi;
    const GemmProblem& q = p.prob[pi];
    const int lt = t - q.tile_begin;
    const int mat = lt / q.tiles_per_mat;
    const int r = lt - mat * q.tiles_per_mat;
    const int tm = r / q.tiles_n, tn = r - (r / q.tiles_n) * q.tiles_n;
    const float* A = static_cast<const float*>(q.a) + mat * q.a_bs;
    const float* B = static_cast<const float*>(q.b) + mat * q.b_bs;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < q.K; k0 += ST_BK) {
      __syncthreads();
      for (int e = threadIdx.x; e < ST_BK * ST_BM; e += 256) {
        const int kk = e / ST_BM, ii = e % ST_BM;
        As[kk][ii] = op_load(A, q.a_ld, q.a_mn, tm * ST_BM + ii, k0 + kk, q.M, q.K);
        Bs[kk][ii] = op_load(B, q.b_ld, q.b_mn, tn * ST_BN + ii, k0 + kk, q.N, q.K);
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < ST_BK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = As[kk][ty * 4 + u], b[u] = Bs[kk][tx * 4 + u];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
      }
    }
    float f = 1.f;
    if (q.scale_mode) {
      const float s = p.scales[q.scale_base + mat];
      f = (q.scale_mode == 1) ? s * s : s;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = tm * ST_BM + ty * 4 + u;
      if (i >= q.M) continue;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int j = tn * ST_BN + tx * 4 + v;
        if (j >= q.N) continue;
        float val = acc[u][v];
        const long long eo = static_cast<long long>(i) * q.ein_ld + j;
        if (EPI == EPI_GRAM) {
          val *= f;
        } else if (EPI == EPI_POLY) {
          const float a = static_cast<const float*>(q.ein)[mat * q.ein_bs + eo];
          val = fmaf(q.cb, a, q.cc * val) + (i == j ? q.ca : 0.f);
        } else {
          val *= f;
        }
        if (EPI == EPI_AXPY_UPDATE) {
          const int wi = q.w_first + mat;
          float* w = p.wptr[wi] + static_cast<long long>(i) * p.wcols[wi] + j;
          *w = cautious_w_f32(*w, val, p.sched ? q.lr * p.sched->lr_mult : q.lr, p.wd, p.cautious != 0);
        } else {
          static_cast<float*>(q.out)[mat * q.out_bs + static_cast<long long>(i) * q.out_ld + j] = val;
        }
      }
    }
  }
}

int simt_tile() { return ST_BM; }

cudaError_t launch_simt_gemm(const SimtGemmParams& p, int epi, int num_sms, cudaStream_t s) {
  if (p.total_tiles <= 0) return cudaSuccess;
  const int grid = p.total_tiles < num_sms * 8 ? p.total_tiles : num_sms * 8;
  switch (epi) {
    case EPI_GRAM: return launch_pdl(simt_gemm_kernel<EPI_GRAM>, dim3(grid), dim3(256), 0, s, p);
    case EPI_POLY: return launch_pdl(simt_gemm_kernel<EPI_POLY>, dim3(grid), dim3(256), 0, s, p);
    case EPI_AXPY: return launch_pdl(simt_gemm_kernel<EPI_AXPY>, dim3(grid), dim3(256), 0, s, p);
    case EPI_AXPY_UPDATE: return launch_pdl(simt_gemm_kernel<EPI_AXPY_UPDATE>, dim3(grid), dim3(256), 0, s, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
