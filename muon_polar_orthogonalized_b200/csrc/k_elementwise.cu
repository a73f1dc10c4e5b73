// k_elementwise.cu -- the HBM-bound kernels of the Muon + AdamW step.
//
//   momentum_norm  m <- beta*m + G;  m~ <- beta*m + G (Nesterov) or m;
//                  X0 <- m~ stored in the workspace (bf16, or fp32 in debug
//                  mode) and one partial sum of m~^2 per block.
//                  ("Chapter 4: The MuonAdamW Optimizer", The Muon Update Rule)
//   momentum_rowq  the same momentum, then MuonEq row equilibration: every
//                  parameter row of m~ divided by (||row|| + 1e-7) before it
//                  is stored as X0; one partial sum per row
//                  (nanochat discussion, mira687's reply: MuonEq)
//   norm_finalize  s <- 1 / (sqrt(sum of partials) + 1e-7), one block per
//                  matrix, fixed summation order (deterministic).
//                  ("Chapter 4", Polar Express: X / (||X|| + 1e-7))
//   update         W <- W - lr*(U + wd*mask*W), mask = (U*W >= 0) by sign bits
//                  (nanochat discussion, mira687's reply: cautious weight decay)
//   emit           out <- U as fp32 (orthogonaliser entry point)
//   normuon_update NorMuon + cautious update, one warp per row: U_row is divided
//                  by (||U_row||/sqrt(cols) + 1e-8) first ("Chapter 4", NorMuon)
//   adamw          bias-corrected AdamW with decoupled decay
//                  ("3.9 Optimizers", Implementing AdamW from scratch)
//
// All of them stream: 16-byte vector accesses where the matrix allows it,
// several independent loads in flight per thread, one chunk per block.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "elt_params.cuh"
#include "pdl.cuh"
#include "sm100.cuh"

namespace muon {

// Launch shapes: the momentum / update kernels stream 2-3 arrays and run
// best at full occupancy (8 x 256 threads per SM) with 2 vec4 units per
// thread (measured on B200, isolated, 1G elements).  AdamW streams 4 arrays;
// with its approximate square root and division it needs 32 registers at 2
// units per thread and full occupancy, with nothing in local memory.
#ifndef MUON_ELT_UNROLL
#define MUON_ELT_UNROLL 2
#endif
#ifndef MUON_ELT_MIN_BLOCKS
#define MUON_ELT_MIN_BLOCKS 8
#endif
#ifndef MUON_ADAM_UNROLL
#define MUON_ADAM_UNROLL 2
#endif
#ifndef MUON_ADAM_MIN_BLOCKS
#define MUON_ADAM_MIN_BLOCKS 8
#endif
constexpr int kEltThreads = 256;
constexpr int kEltUnroll = MUON_ELT_UNROLL;                  // vec4 units per thread
constexpr int kEltMinBlocks = MUON_ELT_MIN_BLOCKS;           // resident blocks per SM (occupancy)
constexpr int kEltChunk = kEltThreads * kEltUnroll * 4;      // elements per work chunk
constexpr int kAdamUnroll = MUON_ADAM_UNROLL;
constexpr int kAdamMinBlocks = MUON_ADAM_MIN_BLOCKS;
constexpr int kAdamChunk = kEltThreads * kAdamUnroll * 4;

// Streaming accesses (each element read and written once per step).
#ifndef MUON_ELT_STREAM_HINTS
#define MUON_ELT_STREAM_HINTS 0
#endif
template <typename T>
__device__ __forceinline__ T ld_stream(const T* p) {
#if MUON_ELT_STREAM_HINTS
  return __ldcs(p);
#else
  return *p;
#endif
}
template <typename T>
__device__ __forceinline__ void st_stream(T* p, T v) {
#if MUON_ELT_STREAM_HINTS
  __stcs(p, v);
#else
  *p = v;
#endif
}

__device__ __forceinline__ int find_mat(const MatRef* mats, int n, int blk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (mats[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float round_bf16(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// Load 4 consecutive gradient values as fp32.
template <bool BF16>
__device__ __forceinline__ float4 load_g4(const void* g, long long e) {
  if constexpr (BF16) {
    uint2 raw = ld_stream(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(g) + e));
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  } else {
    return ld_stream(reinterpret_cast<const float4*>(static_cast<const float*>(g) + e));
  }
}
template <bool BF16>
__device__ __forceinline__ float load_g1(const void* g, long long e) {
  if constexpr (BF16) return bf16_to_f(static_cast<const __nv_bfloat16*>(g)[e]);
  else return static_cast<const float*>(g)[e];
}

__device__ __forceinline__ void store_x4(void* x, long long idx, float4 v, bool f32) {
  if (f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(x) + idx) = v;
  } else {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t*>(&a);
    raw.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(x) + idx) = raw;
  }
}
__device__ __forceinline__ void store_x1(void* x, long long idx, float v, bool f32) {
  if (f32) static_cast<float*>(x)[idx] = v;
  else static_cast<__nv_bfloat16*>(x)[idx] = __float2bfloat16_rn(v);
}
__device__ __forceinline__ float4 load_x4(const void* x, long long idx, bool f32) {
  if (f32) return *reinterpret_cast<const float4*>(static_cast<const float*>(x) + idx);
  uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(x) + idx);
  float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.x));
  float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float load_x1(const void* x, long long idx, bool f32) {
  if (f32) return static_cast<const float*>(x)[idx];
  return bf16_to_f(static_cast<const __nv_bfloat16*>(x)[idx]);
}

// Deterministic block sum (fixed shuffle tree, then warp 0 in order).
__device__ __forceinline__ float block_sum(float v) {
  __shared__ float red[kEltThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  if (w == 0) {
    s = (l < kEltThreads / 32) ? red[l] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  return s;  // valid in thread 0
}

// ------------------------------------------------------------ momentum_norm
// X index of flat element e (multiple of 4 on the vector path): the X buffer
// has pitch ldx >= cols; when they are equal it is e itself.
__device__ __forceinline__ long long x_index(const MatRef& r, long long e) {
  if (r.ldx == r.cols) return e;
  const int ei = static_cast<int>(e);  // numel < 2^31 (checked on the host)
  const int row = ei / r.cols;
  return static_cast<long long>(row) * r.ldx + (ei - row * r.cols);
}

template <bool GBF16>
__device__ __forceinline__ float momentum_chunk(const EltParams& p, const MatRef& r, long long e0) {
  const long long numel = static_cast<long long>(r.rows) * r.cols;
  const float beta = p.beta;
  const bool f32x = p.x_f32 != 0;
  float acc = 0.f;
  if (r.vec) {
    float4 gv[kEltUnroll], mv[kEltUnroll];
#pragma unroll
    for (int u = 0; u < kEltUnroll; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < numel) {
        gv[u] = load_g4<GBF16>(r.g, e);
        mv[u] = r.m ? ld_stream(reinterpret_cast<const float4*>(r.m + e)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kEltUnroll; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < numel) {
        float4 mt;
        if (r.m) {
          float4 mn;
          mn.x = fmaf(beta, mv[u].x, gv[u].x);
          mn.y = fmaf(beta, mv[u].y, gv[u].y);
          mn.z = fmaf(beta, mv[u].z, gv[u].z);
          mn.w = fmaf(beta, mv[u].w, gv[u].w);
          st_stream(reinterpret_cast<float4*>(r.m + e), mn);
          if (p.nesterov) {
            mt.x = fmaf(beta, mn.x, gv[u].x);
            mt.y = fmaf(beta, mn.y, gv[u].y);
            mt.z = fmaf(beta, mn.z, gv[u].z);
            mt.w = fmaf(beta, mn.w, gv[u].w);
          } else {
            mt = mn;
          }
        } else {
          mt = gv[u];
        }
        acc = fmaf(mt.x, mt.x, acc);
        acc = fmaf(mt.y, mt.y, acc);
        acc = fmaf(mt.z, mt.z, acc);
        acc = fmaf(mt.w, mt.w, acc);
        store_x4(r.x, x_index(r, e), mt, f32x);
      }
    }
  } else {
    for (int u = 0; u < kEltUnroll * 4; ++u) {
      const long long e = e0 + static_cast<long long>(u) * kEltThreads + threadIdx.x;
      if (e < numel) {
        const float g = load_g1<GBF16>(r.g, e);
        float mt = g;
        if (r.m) {
          const float mn = fmaf(beta, r.m[e], g);
          r.m[e] = mn;
          mt = p.nesterov ? fmaf(beta, mn, g) : mn;
        }
        acc = fmaf(mt, mt, acc);
        store_x1(r.x, x_index(r, e), mt, f32x);
      }
    }
  }
  return acc;
}

// Persistent: block b handles chunks b, b + grid, ...; every chunk's partial
// sum is reduced in a fixed order, so results do not depend on the grid.
template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads, kEltMinBlocks)
momentum_norm_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  for (int blk = blockIdx.x; blk < p.total_blocks; blk += gridDim.x) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, blk)];
    const long long e0 = static_cast<long long>(blk - r.blk_begin) * kEltChunk;
    const float acc = momentum_chunk<GBF16>(p, r, e0);
    const float s = block_sum(acc);
    if (threadIdx.x == 0) p.partials[blk] = s;
    __syncthreads();  // block_sum's shared scratch is reused by the next chunk
  }
}

// ------------------------------------------------------------ momentum_bulk
// The same update as momentum_norm_kernel, streamed through shared memory by
// the bulk-copy engine: per stage one thread loads two chunks (4096
// elements) of m and G into a 3-stage ring and stores the new m and X0 back
// from it, while all threads compute in shared memory; three blocks per SM
// (measured in the power-capped step of 32 layers: 15.4-17.3 ms against
// 19.1-22.8 ms with two blocks of three or four stages or four of two).  With the copies off
// the load/store units the stream keeps its HBM rate when the SM clock drops
// under the board's power cap (measured on 16 x 4096^2 bf16 gradients:
// 6.25-6.30 TB/s at 1275-1374 MHz, against 5.44-5.58 TB/s for
// momentum_norm_kernel and 5.5 TB/s for a plain float4 copy at those
// clocks).  Each thread handles the elements it would in momentum_norm_kernel
// and sums them in the same order, so m, X0 and every chunk's partial sum
// are bitwise the same.  The host uses it where every matrix of the launch
// has momentum, a bf16 X0 of pitch cols, 16-byte aligned G, m and X0, and a
// multiple of 8 elements.
constexpr int kBulkChunks = 2;                        // chunks per stage
constexpr int kBulkElems = kBulkChunks * kEltChunk;   // 4096
#ifndef MUON_BULK_STAGES
#define MUON_BULK_STAGES 3
#endif
#ifndef MUON_BULK_BLOCKS
#define MUON_BULK_BLOCKS 3
#endif
constexpr int kBulkStages = MUON_BULK_STAGES;
constexpr int kBulkBlocks = MUON_BULK_BLOCKS;         // resident blocks per SM
template <bool GBF16>
struct BulkCfg {
  static constexpr int GSZ = GBF16 ? 2 : 4;
  static constexpr int M_BYTES = kBulkElems * 4;
  static constexpr int STAGE = M_BYTES + kBulkElems * GSZ;   // m, then G (X0 written over G's first bytes)
  static constexpr int SMEM = kBulkStages * STAGE + 64;      // + the stages' mbarriers
};

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads, kBulkBlocks)
momentum_bulk_kernel(const __grid_constant__ EltParams p) {
  using B = BulkCfg<GBF16>;
  extern __shared__ __align__(128) uint8_t bulk_smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(bulk_smem + kBulkStages * B::STAGE);
  __shared__ int abort_flag;
  // item k of this block: its matrix, first chunk, first element, size and
  // the index of its first chunk's partial; written by the loading thread
  // with the stage, so the others read it rather than search the matrices
  struct Item { float* m; __nv_bfloat16* x; int ne, pidx; };
  __shared__ Item stage_item[kBulkStages];
  __shared__ int item_begin[kMaxMatsPerLaunch];   // the matrices' first items, searched per item
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < p.nmats; i += blockDim.x) item_begin[i] = p.mats[i].item_begin;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kBulkStages; ++s) sm100::mbar_init(&full[s], 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const int mine = static_cast<int>(blockIdx.x) < p.total_items
                       ? (p.total_items - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x : 0;
  // load item k into its stage (the loading thread only)
  auto issue = [&](int k) {
    const int it = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    int lo = 0, hi = p.nmats - 1;   // the matrix holding item `it`
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (item_begin[mid] <= it) lo = mid; else hi = mid - 1;
    }
    const MatRef& r = p.mats[lo];
    const int c0 = (it - item_begin[lo]) * kBulkChunks;
    const long long e0 = static_cast<long long>(c0) * kEltChunk;
    const long long numel = static_cast<long long>(r.rows) * r.cols;
    Item t;
    t.ne = static_cast<int>(numel - e0 < kBulkElems ? numel - e0 : kBulkElems);
    t.pidx = r.blk_begin + c0;
    t.m = r.m + e0;
    t.x = static_cast<__nv_bfloat16*>(r.x) + e0;
    const int s = k % kBulkStages;
    uint8_t* st = bulk_smem + s * B::STAGE;
    stage_item[s] = t;   // published to the other threads by the barrier's arrival
    sm100::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(t.ne) * (4 + B::GSZ));
    sm100::bulk_load(st, t.m, static_cast<uint32_t>(t.ne) * 4, &full[s]);
    sm100::bulk_load(st + B::M_BYTES, static_cast<const uint8_t*>(r.g) + e0 * B::GSZ,
                     static_cast<uint32_t>(t.ne) * B::GSZ, &full[s]);
  };
  if (threadIdx.x == 0)
    for (int k = 0; k < mine && k < kBulkStages - 1; ++k) issue(k);
  int next = mine < kBulkStages - 1 ? mine : kBulkStages - 1;   // next item to load (every thread tracks it)
  int k = 0;
  for (; k < mine; ++k) {
    const int s = k % kBulkStages;
    uint8_t* st = bulk_smem + s * B::STAGE;
    const bool got = sm100::mbar_wait(&full[s], static_cast<uint32_t>((k / kBulkStages) & 1), &abort_flag);
    if (!__syncthreads_and(got)) {   // the same decision in every thread
      if (threadIdx.x == 0) atomicOr(p.status, kDevTimeout);
      break;
    }
    const Item t = stage_item[s];
    float* sm = reinterpret_cast<float*>(st);
    uint8_t* sg = st + B::M_BYTES;
    float acc[kBulkChunks] = {};
    // one unit: m~ from the staged m and G, the new m written over m, X0
    // (bf16) over the unit's first bytes of the G slot; the sum of squares
    // in momentum_norm_kernel's order
    auto unit = [&](int h, int e, float4 g, float4 m) {
      float4 mn, mt;
      mn.x = fmaf(p.beta, m.x, g.x);
      mn.y = fmaf(p.beta, m.y, g.y);
      mn.z = fmaf(p.beta, m.z, g.z);
      mn.w = fmaf(p.beta, m.w, g.w);
      *reinterpret_cast<float4*>(sm + e) = mn;
      if (p.nesterov) {
        mt.x = fmaf(p.beta, mn.x, g.x);
        mt.y = fmaf(p.beta, mn.y, g.y);
        mt.z = fmaf(p.beta, mn.z, g.z);
        mt.w = fmaf(p.beta, mn.w, g.w);
      } else {
        mt = mn;
      }
      acc[h] = fmaf(mt.x, mt.x, acc[h]);
      acc[h] = fmaf(mt.y, mt.y, acc[h]);
      acc[h] = fmaf(mt.z, mt.z, acc[h]);
      acc[h] = fmaf(mt.w, mt.w, acc[h]);
      const __nv_bfloat162 a = __floats2bfloat162_rn(mt.x, mt.y);
      const __nv_bfloat162 b = __floats2bfloat162_rn(mt.z, mt.w);
      *reinterpret_cast<uint2*>(sg + e * 2) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
    };
    if constexpr (GBF16) {
      // X0 takes exactly the unit's own G bytes: read and overwrite in place
#pragma unroll
      for (int h = 0; h < kBulkChunks; ++h)
#pragma unroll
        for (int u = 0; u < kEltUnroll; ++u) {
          const int e = h * kEltChunk + (u * kEltThreads + static_cast<int>(threadIdx.x)) * 4;
          if (e < t.ne) {
            const uint2 raw = *reinterpret_cast<const uint2*>(sg + e * 2);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
            unit(h, e, make_float4(a.x, a.y, b.x, b.y), *reinterpret_cast<const float4*>(sm + e));
          }
        }
    } else {
      // fp32 G: X0 (2 bytes per element) overlaps other threads' G, so every
      // unit is read before any is written
      float4 gv[kBulkChunks][kEltUnroll], mv[kBulkChunks][kEltUnroll];
#pragma unroll
      for (int h = 0; h < kBulkChunks; ++h)
#pragma unroll
        for (int u = 0; u < kEltUnroll; ++u) {
          const int e = h * kEltChunk + (u * kEltThreads + static_cast<int>(threadIdx.x)) * 4;
          if (e < t.ne) {
            gv[h][u] = *reinterpret_cast<const float4*>(sg + e * 4);
            mv[h][u] = *reinterpret_cast<const float4*>(sm + e);
          }
        }
      __syncthreads();
#pragma unroll
      for (int h = 0; h < kBulkChunks; ++h)
#pragma unroll
        for (int u = 0; u < kEltUnroll; ++u) {
          const int e = h * kEltChunk + (u * kEltThreads + static_cast<int>(threadIdx.x)) * 4;
          if (e < t.ne) unit(h, e, gv[h][u], mv[h][u]);
        }
    }
    sm100::fence_proxy_async_smem();   // the generic-proxy writes above, for the bulk stores
    __syncthreads();
    if (threadIdx.x == 0) {
      sm100::bulk_store(t.m, sm, static_cast<uint32_t>(t.ne) * 4);
      sm100::bulk_store(t.x, sg, static_cast<uint32_t>(t.ne) * 2);
      sm100::bulk_commit_group();
      if (next < mine) {
        sm100::bulk_wait_group_read<1>();   // the stage stored one item ago may be refilled
        issue(next);
      }
    }
    if (next < mine) ++next;
    // the partial sum of each of the item's chunks
    const int nch = (t.ne + kEltChunk - 1) / kEltChunk;
#pragma unroll
    for (int h = 0; h < kBulkChunks; ++h) {
      const float tot = block_sum(acc[h]);
      if (threadIdx.x == 0 && h < nch) p.partials[t.pidx + h] = tot;
      __syncthreads();   // block_sum's shared scratch is reused
    }
  }
  if (threadIdx.x == 0) {
    sm100::bulk_wait_group<0>();   // every store written
    // after a timeout: loads issued but not consumed land before the block
    // exits (each wait bounded)
    for (int j = k; j < next; ++j) {
      const uint64_t t0 = sm100::globaltimer();
      while (!sm100::mbar_try_wait(&full[j % kBulkStages], static_cast<uint32_t>((j / kBulkStages) & 1)) &&
             sm100::globaltimer() - t0 < 100000000ull) {
      }
    }
  }
}

// ------------------------------------------------------------ momentum_rowq
// MuonEq: the momentum update, then every parameter row of m~ divided by
// (||row|| + 1e-7) as it is stored as X0.  Each row's partial is
// (||m~_row|| f)^2 with f = 1/(||m~_row|| + 1e-7), the squared norm of the
// equilibrated row, stored at partials[pbase + row]; norm_finalize then
// yields the Frobenius scale of the equilibrated matrix.  Rows are numbered
// consecutively over the matrices of a launch (MatRef.blk_begin = first row).
// Row sums of squares are taken in a fixed order.  The host sorts rows into
// four launches by width, so that each keeps enough loads in flight:
//   rowq_warp   vector rows of <= 768 columns: one warp per row, m~ in
//               registers (6 float4 per lane), shuffle reduction;
//   rowq_block  vector rows of <= 4096 columns: one block per row, m~ in
//               registers (4 float4 per thread);
//   momentum_rowq_kernel, vector rows of <= 16384 columns: one block per row,
//               m~ in dynamic shared memory (each thread reads back only the
//               entries it wrote);
//   momentum_rowq_kernel, longer or unaligned rows: pass 2 recomputes m~ from
//               G and the momentum this thread just wrote (the same fp32
//               operations, so the same values).
constexpr int kRowEqWarpCols = 768;                       // 32 lanes x 6 float4
constexpr int kRowEqWarpVec = kRowEqWarpCols / 128;
constexpr int kRowEqBlockVec = 4;
constexpr int kRowEqBlockCols = kEltThreads * 4 * kRowEqBlockVec;  // 4096
constexpr int kRowEqSmemCols = 16384;
constexpr int kRowEqUnroll = 4;  // float4 units in flight per thread (shared-memory path)
constexpr float kRowEqEps = 1e-7f;

__device__ __forceinline__ float4 momentum4(const EltParams& p, float* m, long long e, float4 g, float4 mv) {
  if (!m) return g;
  float4 mn;
  mn.x = fmaf(p.beta, mv.x, g.x);
  mn.y = fmaf(p.beta, mv.y, g.y);
  mn.z = fmaf(p.beta, mv.z, g.z);
  mn.w = fmaf(p.beta, mv.w, g.w);
  st_stream(reinterpret_cast<float4*>(m + e), mn);
  if (!p.nesterov) return mn;
  return make_float4(fmaf(p.beta, mn.x, g.x), fmaf(p.beta, mn.y, g.y), fmaf(p.beta, mn.z, g.z),
                     fmaf(p.beta, mn.w, g.w));
}
// m~ again from G and the momentum already written by momentum4
__device__ __forceinline__ float4 lookahead4(const EltParams& p, const float* m, long long e, float4 g) {
  if (!m) return g;
  const float4 mn = *reinterpret_cast<const float4*>(m + e);
  if (!p.nesterov) return mn;
  return make_float4(fmaf(p.beta, mn.x, g.x), fmaf(p.beta, mn.y, g.y), fmaf(p.beta, mn.z, g.z),
                     fmaf(p.beta, mn.w, g.w));
}
__device__ __forceinline__ float sumsq4(float4 v, float acc) {
  acc = fmaf(v.x, v.x, acc);
  acc = fmaf(v.y, v.y, acc);
  acc = fmaf(v.z, v.z, acc);
  return fmaf(v.w, v.w, acc);
}
__device__ __forceinline__ float4 scale4(float4 v, float f) {
  return make_float4(v.x * f, v.y * f, v.z * f, v.w * f);
}
__device__ __forceinline__ float4 load_m4(const float* m, long long e) {
  return m ? ld_stream(reinterpret_cast<const float4*>(m + e)) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// Loads NV float4 units of one row (unit u at column base + u*stride + lane4),
// runs the momentum update, keeps m~ in `keep` and returns this thread's sum
// of squares (units in order).
template <bool GBF16, int NV>
__device__ __forceinline__ float rowq_load_regs(const EltParams& p, const MatRef& r, long long e0,
                                                int first, int stride, float4 (&keep)[NV]) {
  float4 gv[NV];
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int c = first + u * stride;
    if (c < r.cols) {
      gv[u] = load_g4<GBF16>(r.g, e0 + c);
      keep[u] = load_m4(r.m, e0 + c);
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int c = first + u * stride;
    if (c < r.cols) {
      keep[u] = momentum4(p, r.m, e0 + c, gv[u], keep[u]);
      acc = sumsq4(keep[u], acc);
    }
  }
  return acc;
}

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads, 3)
rowq_warp_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int wpb = kEltThreads / 32;
  const bool f32x = p.x_f32 != 0;
  for (int row_g = blockIdx.x * wpb + static_cast<int>(threadIdx.x >> 5); row_g < p.total_blocks;
       row_g += gridDim.x * wpb) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, row_g)];
    const int row = row_g - r.blk_begin;
    const long long e0 = static_cast<long long>(row) * r.cols;
    float4 keep[kRowEqWarpVec];
    float acc = rowq_load_regs<GBF16, kRowEqWarpVec>(p, r, e0, lane * 4, 128, keep);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const float nrm = sqrtf(acc);
    const float f = 1.f / (nrm + kRowEqEps);
    if (lane == 0) {
      const float q = nrm * f;
      p.partials[r.pbase + row] = q * q;
    }
    const long long x0 = static_cast<long long>(row) * r.ldx;
#pragma unroll
    for (int u = 0; u < kRowEqWarpVec; ++u) {
      const int c = lane * 4 + u * 128;
      if (c < r.cols) store_x4(r.x, x0 + c, scale4(keep[u], f), f32x);
    }
  }
}

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads)
rowq_block_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float row_ss;
  const bool f32x = p.x_f32 != 0;
  for (int row_g = blockIdx.x; row_g < p.total_blocks; row_g += gridDim.x) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, row_g)];
    const int row = row_g - r.blk_begin;
    const long long e0 = static_cast<long long>(row) * r.cols;
    float4 keep[kRowEqBlockVec];
    const float acc = rowq_load_regs<GBF16, kRowEqBlockVec>(p, r, e0, static_cast<int>(threadIdx.x) * 4,
                                                            kEltThreads * 4, keep);
    const float tot = block_sum(acc);
    if (threadIdx.x == 0) row_ss = tot;
    __syncthreads();
    const float nrm = sqrtf(row_ss);
    const float f = 1.f / (nrm + kRowEqEps);
    if (threadIdx.x == 0) {
      const float q = nrm * f;
      p.partials[r.pbase + row] = q * q;
    }
    const long long x0 = static_cast<long long>(row) * r.ldx;
#pragma unroll
    for (int u = 0; u < kRowEqBlockVec; ++u) {
      const int c = static_cast<int>(threadIdx.x) * 4 + u * kEltThreads * 4;
      if (c < r.cols) store_x4(r.x, x0 + c, scale4(keep[u], f), f32x);
    }
  }
}

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads)
momentum_rowq_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ float4 rowbuf[];  // kRowEqSmemCols / 4 entries at most
  __shared__ float row_ss;
  const bool f32x = p.x_f32 != 0;
  constexpr int kStep = kEltThreads * 4;  // columns per unit
  for (int row_g = blockIdx.x; row_g < p.total_blocks; row_g += gridDim.x) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, row_g)];
    const int row = row_g - r.blk_begin;
    const long long e0 = static_cast<long long>(row) * r.cols;
    const long long x0 = static_cast<long long>(row) * r.ldx;
    const bool in_smem = r.vec && r.cols <= kRowEqSmemCols;
    float acc = 0.f;
    if (r.vec) {
      for (int base = 0; base < r.cols; base += kStep * kRowEqUnroll) {
        float4 gv[kRowEqUnroll], mv[kRowEqUnroll];
#pragma unroll
        for (int u = 0; u < kRowEqUnroll; ++u) {
          const int c = base + u * kStep + static_cast<int>(threadIdx.x) * 4;
          if (c < r.cols) {
            gv[u] = load_g4<GBF16>(r.g, e0 + c);
            mv[u] = load_m4(r.m, e0 + c);
          }
        }
#pragma unroll
        for (int u = 0; u < kRowEqUnroll; ++u) {
          const int c = base + u * kStep + static_cast<int>(threadIdx.x) * 4;
          if (c < r.cols) {
            const float4 mt = momentum4(p, r.m, e0 + c, gv[u], mv[u]);
            acc = sumsq4(mt, acc);
            if (in_smem) rowbuf[c >> 2] = mt;
          }
        }
      }
    } else {
      for (int c = threadIdx.x; c < r.cols; c += kEltThreads) {
        const float g = load_g1<GBF16>(r.g, e0 + c);
        float mt = g;
        if (r.m) {
          const float mn = fmaf(p.beta, r.m[e0 + c], g);
          r.m[e0 + c] = mn;
          mt = p.nesterov ? fmaf(p.beta, mn, g) : mn;
        }
        acc = fmaf(mt, mt, acc);
      }
    }
    const float tot = block_sum(acc);
    if (threadIdx.x == 0) row_ss = tot;
    __syncthreads();
    const float nrm = sqrtf(row_ss);
    const float f = 1.f / (nrm + kRowEqEps);
    if (threadIdx.x == 0) {
      const float q = nrm * f;
      p.partials[r.pbase + row] = q * q;
    }
    if (in_smem) {
      for (int c = threadIdx.x * 4; c < r.cols; c += kStep)
        store_x4(r.x, x0 + c, scale4(rowbuf[c >> 2], f), f32x);
    } else if (r.vec) {
      for (int c = threadIdx.x * 4; c < r.cols; c += kStep) {
        const float4 g = load_g4<GBF16>(r.g, e0 + c);
        store_x4(r.x, x0 + c, scale4(lookahead4(p, r.m, e0 + c, g), f), f32x);
      }
    } else {
      for (int c = threadIdx.x; c < r.cols; c += kEltThreads) {
        const float g = load_g1<GBF16>(r.g, e0 + c);
        float mt = g;
        if (r.m) {
          const float mn = r.m[e0 + c];
          mt = p.nesterov ? fmaf(p.beta, mn, g) : mn;
        }
        store_x1(r.x, x0 + c, mt * f, f32x);
      }
    }
  }
}

// ------------------------------------------------------------ norm_finalize
// Sums the matrix's partials (one per momentum block, or one per row with
// MuonEq) in fp64 in a fixed order.
__global__ void __launch_bounds__(kEltThreads)
norm_finalize_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const MatRef& r = p.mats[blockIdx.x];
  const long long numel = static_cast<long long>(r.rows) * r.cols;
  const int nblk = p.row_eq ? r.rows : static_cast<int>((numel + kEltChunk - 1) / kEltChunk);
  double acc = 0.0;
  for (int i = threadIdx.x; i < nblk; i += kEltThreads) acc += p.partials[r.blk_begin + i];
  __shared__ double red[kEltThreads];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = kEltThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) p.scales[r.sidx] = static_cast<float>(1.0 / (sqrt(red[0]) + 1e-7));
}

// --------------------------------------------------------- update / emit
// U = X (bf16 values, or fp32 in debug mode), times the matrix scale when no
// Newton-Schulz step ran; the bf16 path rounds that product to bf16 as the
// pages' bf16 X would be.
__device__ __forceinline__ float cautious_apply(float w, float u, float lr, float wd,
                                                bool cautious) {
  // mask = (u*w >= 0) decided from sign bits: equal signs, or either is zero
  bool mask = true;
  if (cautious) {
    const bool sdiff = (__float_as_uint(u) ^ __float_as_uint(w)) >> 31;
    mask = !sdiff || u == 0.f || w == 0.f;
  }
  const float t = mask ? fmaf(wd, w, u) : u;
  return fmaf(-lr, t, w);
}

template <bool EMIT>
__device__ __forceinline__ void update_chunk(const EltParams& p, const MatRef& r, long long e0) {
  const long long numel = static_cast<long long>(r.rows) * r.cols;
  const float lr = p.sched ? r.lr * p.sched->lr_mult : r.lr;
  const bool f32x = p.x_f32 != 0;
  const float sc = p.use_scale ? p.scales[r.sidx] : 1.f;
  auto make_u = [&](float x) {
    if (!p.use_scale) return x;
    return f32x ? sc * x : round_bf16(sc * x);
  };
  if (r.vec) {
    float4 xv[kEltUnroll], wv[kEltUnroll];
#pragma unroll
    for (int u = 0; u < kEltUnroll; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < numel) {
        xv[u] = load_x4(r.x, x_index(r, e), f32x);
        if (!EMIT) wv[u] = ld_stream(reinterpret_cast<const float4*>(r.w + e));
      }
    }
#pragma unroll
    for (int u = 0; u < kEltUnroll; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < numel) {
        float4 uu = make_float4(make_u(xv[u].x), make_u(xv[u].y), make_u(xv[u].z), make_u(xv[u].w));
        if (EMIT) {
          st_stream(reinterpret_cast<float4*>(r.out + e), uu);
        } else {
          float4 w = wv[u];
          w.x = cautious_apply(w.x, uu.x, lr, p.wd, p.cautious);
          w.y = cautious_apply(w.y, uu.y, lr, p.wd, p.cautious);
          w.z = cautious_apply(w.z, uu.z, lr, p.wd, p.cautious);
          w.w = cautious_apply(w.w, uu.w, lr, p.wd, p.cautious);
          st_stream(reinterpret_cast<float4*>(r.w + e), w);
        }
      }
    }
  } else {
    for (int u = 0; u < kEltUnroll * 4; ++u) {
      const long long e = e0 + static_cast<long long>(u) * kEltThreads + threadIdx.x;
      if (e < numel) {
        const float uu = make_u(load_x1(r.x, x_index(r, e), f32x));
        if (EMIT) r.out[e] = uu;
        else r.w[e] = cautious_apply(r.w[e], uu, lr, p.wd, p.cautious);
      }
    }
  }
}

template <bool EMIT>
__global__ void __launch_bounds__(kEltThreads, kEltMinBlocks)
update_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  for (int blk = blockIdx.x; blk < p.total_blocks; blk += gridDim.x) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, blk)];
    update_chunk<EMIT>(p, r, static_cast<long long>(blk - r.blk_begin) * kEltChunk);
  }
}

// -------------------------------------------------------- normuon_update
// NorMuon + cautious update, one warp per parameter row (rows of all matrices
// of the launch are numbered consecutively: MatRef.blk_begin = first row).
// Pass 1 sums U^2 over the row (U = the bf16 X, or bf16(s*X0) when no
// iteration ran) in fp32 per lane in column order, reduced by a fixed shuffle
// tree; f = 1/(sqrt(sum/cols) + 1e-8).  Pass 2 re-reads the row (now in
// cache) and applies W <- W - lr*(f*U + wd*mask*W).
__device__ __forceinline__ void ld_x8(const void* x, long long idx, bool f32, float (&v)[8]) {
  if (f32) {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(x) + idx);
    const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(x) + idx + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 raw = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + idx);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
      v[2 * h] = f.x;
      v[2 * h + 1] = f.y;
    }
  }
}

__global__ void __launch_bounds__(kEltThreads)
normuon_update_kernel(const __grid_constant__ EltParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int wpb = kEltThreads / 32;
  const bool f32x = p.x_f32 != 0;
  for (int row_g = blockIdx.x * wpb + (threadIdx.x >> 5); row_g < p.total_blocks;
       row_g += gridDim.x * wpb) {
    const MatRef& r = p.mats[find_mat(p.mats, p.nmats, row_g)];
    const int row = row_g - r.blk_begin;
    const float sc = p.use_scale ? p.scales[r.sidx] : 1.f;
    auto make_u = [&](float x) {
      if (!p.use_scale) return x;
      return f32x ? sc * x : round_bf16(sc * x);
    };
    const long long xb = static_cast<long long>(row) * r.ldx;
    float* wrow = r.w + static_cast<long long>(row) * r.cols;
    const float lr = p.sched ? r.lr * p.sched->lr_mult : r.lr;
    // r.vec: cols % 8 == 0 and W 16-byte aligned (X rows always are)
    float acc = 0.f;
    if (r.vec) {
      for (int c = lane * 8; c < r.cols; c += 256) {
        float v[8];
        ld_x8(r.x, xb + c, f32x, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float u = make_u(v[k]);
          acc = fmaf(u, u, acc);
        }
      }
    } else {
      for (int c = lane; c < r.cols; c += 32) {
        const float u = make_u(load_x1(r.x, xb + c, f32x));
        acc = fmaf(u, u, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const float f = 1.f / (sqrtf(acc / static_cast<float>(r.cols)) + 1e-8f);
    if (r.vec) {
      for (int c = lane * 8; c < r.cols; c += 256) {
        float v[8];
        ld_x8(r.x, xb + c, f32x, v);
        float4* w4 = reinterpret_cast<float4*>(wrow + c);
        float4 w0 = w4[0], w1 = w4[1];
        w0.x = cautious_apply(w0.x, f * make_u(v[0]), lr, p.wd, p.cautious);
        w0.y = cautious_apply(w0.y, f * make_u(v[1]), lr, p.wd, p.cautious);
        w0.z = cautious_apply(w0.z, f * make_u(v[2]), lr, p.wd, p.cautious);
        w0.w = cautious_apply(w0.w, f * make_u(v[3]), lr, p.wd, p.cautious);
        w1.x = cautious_apply(w1.x, f * make_u(v[4]), lr, p.wd, p.cautious);
        w1.y = cautious_apply(w1.y, f * make_u(v[5]), lr, p.wd, p.cautious);
        w1.z = cautious_apply(w1.z, f * make_u(v[6]), lr, p.wd, p.cautious);
        w1.w = cautious_apply(w1.w, f * make_u(v[7]), lr, p.wd, p.cautious);
        w4[0] = w0;
        w4[1] = w1;
      }
    } else {
      for (int c = lane; c < r.cols; c += 32)
        wrow[c] = cautious_apply(wrow[c], f * make_u(load_x1(r.x, xb + c, f32x)), lr, p.wd, p.cautious);
    }
  }
}

// ------------------------------------------------------------------ AdamW
__device__ __forceinline__ int find_tensor(const AdamTensor* t, int n, int blk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (t[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The square root and the division of the step take the hardware's
// approximate forms (sqrt.approx: a few units in the last place; __fdividef:
// 2 ulp for the denominators that occur here, >= eps): each leaves a relative
// error near 1e-7 in the step lr*m/denom, ~1e-9 of p, while the
// correctly-rounded forms cost about four times the instructions, which
// matter at the 1.0-1.3 GHz a power-capped step runs at.  m and v are
// computed exactly as the page's update writes them.
__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void adam_elem(const AdamTensor& T, float g, float& p, float& m,
                                          float& v) {
  p = p * T.decay;
  m = fmaf(T.b1, m, T.omb1 * g);
  v = fmaf(T.b2, v, T.omb2 * (g * g));
  const float denom = fmaf(sqrt_approx(v), T.rsqrt_bc2, T.eps);
  p = fmaf(-T.step_size, __fdividef(m, denom), p);
}

template <bool GBF16>
__device__ __forceinline__ void adamw_chunk(const AdamTensor& T, long long e0) {
  if (T.vec) {
    constexpr int U = kAdamUnroll / 2;  // 4 streams per element: two halves keep registers in check
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float4 gv[U], pv[U], mv[U], vv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const long long e =
            e0 + (static_cast<long long>(half * U + u) * kEltThreads + threadIdx.x) * 4;
        if (e < T.numel) {
          gv[u] = load_g4<GBF16>(T.g, e);
          pv[u] = ld_stream(reinterpret_cast<const float4*>(T.p + e));
          mv[u] = ld_stream(reinterpret_cast<const float4*>(T.m + e));
          vv[u] = ld_stream(reinterpret_cast<const float4*>(T.v + e));
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const long long e =
            e0 + (static_cast<long long>(half * U + u) * kEltThreads + threadIdx.x) * 4;
        if (e < T.numel) {
          adam_elem(T, gv[u].x, pv[u].x, mv[u].x, vv[u].x);
          adam_elem(T, gv[u].y, pv[u].y, mv[u].y, vv[u].y);
          adam_elem(T, gv[u].z, pv[u].z, mv[u].z, vv[u].z);
          adam_elem(T, gv[u].w, pv[u].w, mv[u].w, vv[u].w);
          st_stream(reinterpret_cast<float4*>(T.p + e), pv[u]);
          st_stream(reinterpret_cast<float4*>(T.m + e), mv[u]);
          st_stream(reinterpret_cast<float4*>(T.v + e), vv[u]);
        }
      }
    }
  } else {
    for (int u = 0; u < kAdamUnroll * 4; ++u) {
      const long long e = e0 + static_cast<long long>(u) * kEltThreads + threadIdx.x;
      if (e < T.numel) {
        float pp = T.p[e], mm = T.m[e], vv = T.v[e];
        adam_elem(T, load_g1<GBF16>(T.g, e), pp, mm, vv);
        T.p[e] = pp;
        T.m[e] = mm;
        T.v[e] = vv;
      }
    }
  }
}

// With a device schedule the step-dependent scalars come from the device
// state (lr multiplier, step t), in double like the host path, then fp32.
__device__ __forceinline__ void sched_scalars(AdamTensor& T, const DevSched* s) {
  const double t = static_cast<double>(s->step);
  const double lr = static_cast<double>(T.lr) * static_cast<double>(s->lr_mult);
  T.decay = static_cast<float>(1.0 - lr * static_cast<double>(T.wd));
  T.step_size = static_cast<float>(lr / (1.0 - pow(static_cast<double>(T.b1), t)));
  T.rsqrt_bc2 = static_cast<float>(1.0 / sqrt(1.0 - pow(static_cast<double>(T.b2), t)));
}

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads, kAdamMinBlocks)
adamw_kernel(const __grid_constant__ AdamParams P) {
  pdl_wait();
  pdl_launch_dependents();
  for (int blk = blockIdx.x; blk < P.total_blocks; blk += gridDim.x) {
    const int ti = find_tensor(P.t, P.ntensors, blk);
    if (P.sched) {
      AdamTensor T = P.t[ti];
      sched_scalars(T, P.sched);
      adamw_chunk<GBF16>(T, static_cast<long long>(blk - T.blk_begin) * kAdamChunk);
    } else {
      const AdamTensor& T = P.t[ti];
      adamw_chunk<GBF16>(T, static_cast<long long>(blk - T.blk_begin) * kAdamChunk);
    }
  }
}

// ------------------------------------------------------------- adamw_bulk
// The same update as adamw_kernel, streamed through shared memory by the
// bulk-copy engine like momentum_bulk_kernel: per stage one thread loads a
// 2048-element chunk of g, p, m and v into a ring and stores p, m and v back
// from it; every thread updates its elements in place in shared memory with
// adam_elem, so the results are bitwise those of adamw_kernel.  Used where
// every tensor of the launch has a multiple of 8 elements.
#ifndef MUON_ADAM_BULK_STAGES
#define MUON_ADAM_BULK_STAGES 3
#endif
constexpr int kAdamBulkStages = MUON_ADAM_BULK_STAGES;
template <bool GBF16>
struct AdamBulkCfg {
  static constexpr int GSZ = GBF16 ? 2 : 4;
  static constexpr int P_OFF = 0, M_OFF = kAdamChunk * 4, V_OFF = 2 * kAdamChunk * 4, G_OFF = 3 * kAdamChunk * 4;
  static constexpr int STAGE = 3 * kAdamChunk * 4 + kAdamChunk * GSZ;
  static constexpr int SMEM = kAdamBulkStages * STAGE + 64;   // + the stages' mbarriers
};

// Per device: set when a bounded wait in adamw_bulk_kernel ran out (read and
// cleared by adamw_query_status; AdamW has no caller workspace).
__device__ unsigned int g_adamw_status;

template <bool GBF16>
__global__ void __launch_bounds__(kEltThreads)
adamw_bulk_kernel(const __grid_constant__ AdamParams P) {
  using B = AdamBulkCfg<GBF16>;
  extern __shared__ __align__(128) uint8_t adam_smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(adam_smem + kAdamBulkStages * B::STAGE);
  __shared__ int abort_flag;
  struct Item { int ti, ne; long long e0; };
  __shared__ Item stage_item[kAdamBulkStages];
  __shared__ int blk_begin[kMaxAdamTensors];   // the tensors' first chunks, searched per chunk
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < P.ntensors; i += blockDim.x) blk_begin[i] = P.t[i].blk_begin;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kAdamBulkStages; ++s) sm100::mbar_init(&full[s], 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const int mine = static_cast<int>(blockIdx.x) < P.total_blocks
                       ? (P.total_blocks - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x : 0;
  auto issue = [&](int k) {   // the loading thread only
    const int blk = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    int lo = 0, hi = P.ntensors - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (blk_begin[mid] <= blk) lo = mid; else hi = mid - 1;
    }
    const AdamTensor& T = P.t[lo];
    Item t;
    t.ti = lo;
    t.e0 = static_cast<long long>(blk - blk_begin[lo]) * kAdamChunk;
    t.ne = static_cast<int>(T.numel - t.e0 < kAdamChunk ? T.numel - t.e0 : kAdamChunk);
    const int s = k % kAdamBulkStages;
    uint8_t* st = adam_smem + s * B::STAGE;
    stage_item[s] = t;   // published to the other threads by the barrier's arrival
    const uint32_t ne = static_cast<uint32_t>(t.ne);
    sm100::mbar_arrive_expect_tx(&full[s], ne * (12 + B::GSZ));
    sm100::bulk_load(st + B::P_OFF, T.p + t.e0, ne * 4, &full[s]);
    sm100::bulk_load(st + B::M_OFF, T.m + t.e0, ne * 4, &full[s]);
    sm100::bulk_load(st + B::V_OFF, T.v + t.e0, ne * 4, &full[s]);
    sm100::bulk_load(st + B::G_OFF, static_cast<const uint8_t*>(T.g) + t.e0 * B::GSZ, ne * B::GSZ, &full[s]);
  };
  if (threadIdx.x == 0)
    for (int k = 0; k < mine && k < kAdamBulkStages - 1; ++k) issue(k);
  int next = mine < kAdamBulkStages - 1 ? mine : kAdamBulkStages - 1;   // next chunk to load (every thread tracks it)
  int k = 0;
  for (; k < mine; ++k) {
    const int s = k % kAdamBulkStages;
    uint8_t* st = adam_smem + s * B::STAGE;
    const bool got = sm100::mbar_wait(&full[s], static_cast<uint32_t>((k / kAdamBulkStages) & 1), &abort_flag);
    if (!__syncthreads_and(got)) {   // the same decision in every thread; nothing more is stored
      if (threadIdx.x == 0) atomicOr(&g_adamw_status, kDevTimeout);
      break;
    }
    const Item t = stage_item[s];
    AdamTensor T = P.t[t.ti];
    if (P.sched) sched_scalars(T, P.sched);
    float* sp = reinterpret_cast<float*>(st + B::P_OFF);
    float* smv = reinterpret_cast<float*>(st + B::M_OFF);
    float* svv = reinterpret_cast<float*>(st + B::V_OFF);
#pragma unroll
    for (int u = 0; u < kAdamUnroll; ++u) {
      const int e = (u * kEltThreads + static_cast<int>(threadIdx.x)) * 4;
      if (e < t.ne) {
        float4 g;
        if constexpr (GBF16) {
          const uint2 raw = *reinterpret_cast<const uint2*>(st + B::G_OFF + e * 2);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
          const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
          g = make_float4(a.x, a.y, b.x, b.y);
        } else {
          g = *reinterpret_cast<const float4*>(st + B::G_OFF + e * 4);
        }
        float4 pv = *reinterpret_cast<const float4*>(sp + e);
        float4 mv = *reinterpret_cast<const float4*>(smv + e);
        float4 vv = *reinterpret_cast<const float4*>(svv + e);
        adam_elem(T, g.x, pv.x, mv.x, vv.x);
        adam_elem(T, g.y, pv.y, mv.y, vv.y);
        adam_elem(T, g.z, pv.z, mv.z, vv.z);
        adam_elem(T, g.w, pv.w, mv.w, vv.w);
        *reinterpret_cast<float4*>(sp + e) = pv;
        *reinterpret_cast<float4*>(smv + e) = mv;
        *reinterpret_cast<float4*>(svv + e) = vv;
      }
    }
    sm100::fence_proxy_async_smem();   // the generic-proxy writes above, for the bulk stores
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t ne = static_cast<uint32_t>(t.ne);
      sm100::bulk_store(T.p + t.e0, sp, ne * 4);
      sm100::bulk_store(T.m + t.e0, smv, ne * 4);
      sm100::bulk_store(T.v + t.e0, svv, ne * 4);
      sm100::bulk_commit_group();
      if (next < mine) {
        sm100::bulk_wait_group_read<1>();   // the stage stored one chunk ago may be refilled
        issue(next);
      }
    }
    if (next < mine) ++next;
  }
  if (threadIdx.x == 0) {
    sm100::bulk_wait_group<0>();   // every store written
    // after a timeout: loads issued but not consumed land before the block
    // exits (each wait bounded)
    for (int j = k; j < next; ++j) {
      const uint64_t t0 = sm100::globaltimer();
      while (!sm100::mbar_try_wait(&full[j % kAdamBulkStages], static_cast<uint32_t>((j / kAdamBulkStages) & 1)) &&
             sm100::globaltimer() - t0 < 100000000ull) {
      }
    }
  }
}

// ----------------------------------------------------------- schedule
// step <- step + 1; lr_mult <- trapezoid(step - 1): linear warmup from 0 over
// int(total*warmup_frac) steps, 1 on the flat part, linear warmdown to
// final_frac over int(total*warmdown_frac) steps, final_frac from the end on
// ("Chapter 4: The MuonAdamW Optimizer", trapezoidal schedule).
__global__ void schedule_advance_kernel(DevSched* s, long long total, double warmup_frac,
                                        double warmdown_frac, double final_frac) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const long long t = s->step + 1;
  const long long step = t - 1;
  const long long warm = static_cast<long long>(static_cast<double>(total) * warmup_frac);
  const long long down = static_cast<long long>(static_cast<double>(total) * warmdown_frac);
  const long long flat = total - warm - down;
  double m;
  if (step < warm) m = static_cast<double>(step) / static_cast<double>(warm);
  else if (step < warm + flat) m = 1.0;
  else if (down == 0 || step >= total) m = final_frac;
  else m = final_frac + (1.0 - final_frac) * (1.0 - static_cast<double>(step - warm - flat) / static_cast<double>(down));
  s->step = t;
  s->lr_mult = static_cast<float>(m);
}

// ------------------------------------------------------------- replicate
// dst[r][i] <- src[i]: persistent, 4096-element chunks, 16-byte accesses
// (every pointer is 16-byte aligned; a matrix's scalar tail is copied last).
constexpr int kReplChunk = kEltThreads * 4 * 4;

__global__ void __launch_bounds__(kEltThreads)
replicate_kernel(const __grid_constant__ ReplParams p) {
  pdl_wait();
  pdl_launch_dependents();
  for (int blk = blockIdx.x; blk < p.total_blocks; blk += gridDim.x) {
    int mi = 0;
    while (mi + 1 < p.nmats && p.blk_begin[mi + 1] <= blk) ++mi;
    const long long e0 = static_cast<long long>(blk - p.blk_begin[mi]) * kReplChunk;
    const long long n = p.numel[mi];
    const long long nvec = n & ~3ll;
    const float* src = p.src[mi];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < nvec) {
        const float4 v = *reinterpret_cast<const float4*>(src + e);
        for (int r = 0; r < p.nrep; ++r) *reinterpret_cast<float4*>(p.dst[r][mi] + e) = v;
      }
    }
    if (e0 + kReplChunk >= n && threadIdx.x < n - nvec) {   // the matrix's last chunk: scalar tail
      const long long e = nvec + threadIdx.x;
      for (int r = 0; r < p.nrep; ++r) p.dst[r][mi][e] = src[e];
    }
  }
}

int repl_chunk() { return kReplChunk; }

// ------------------------------------------------------------ reduce_mean
// Persistent, 4096-element chunks; each thread handles 4 groups of 4
// consecutive elements (16-byte fp32 / 8-byte bf16 accesses; every pointer
// is 16-byte aligned), the tail of a tensor element by element.
template <bool BF16>
__global__ void __launch_bounds__(kEltThreads)
reduce_mean_kernel(const __grid_constant__ MeanParams p) {
  pdl_wait();
  pdl_launch_dependents();
  for (int blk = blockIdx.x; blk < p.total_blocks; blk += gridDim.x) {
    int ti = 0;
    while (ti + 1 < p.ntensors && p.blk_begin[ti + 1] <= blk) ++ti;
    const long long e0 = static_cast<long long>(blk - p.blk_begin[ti]) * kReplChunk;
    const long long n = p.numel[ti];
    const long long nvec = n & ~3ll;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long e = e0 + (static_cast<long long>(u) * kEltThreads + threadIdx.x) * 4;
      if (e < nvec) {
        float4 acc = load_g4<BF16>(p.src[0][ti], e);
        for (int r = 1; r < p.nsrc; ++r) {
          const float4 g = load_g4<BF16>(p.src[r][ti], e);
          acc.x += g.x; acc.y += g.y; acc.z += g.z; acc.w += g.w;
        }
        acc.x *= p.inv_n; acc.y *= p.inv_n; acc.z *= p.inv_n; acc.w *= p.inv_n;
        store_x4(p.dst[ti], e, acc, !BF16);
      }
    }
    if (e0 + kReplChunk >= n && threadIdx.x < n - nvec) {   // the tensor's last chunk: scalar tail
      const long long e = nvec + threadIdx.x;
      float acc = load_g1<BF16>(p.src[0][ti], e);
      for (int r = 1; r < p.nsrc; ++r) acc += load_g1<BF16>(p.src[r][ti], e);
      store_x1(p.dst[ti], e, acc * p.inv_n, !BF16);
    }
  }
}

cudaError_t launch_reduce_mean(const MeanParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  const long long g = static_cast<long long>(sms) * 4;
  const int grid = static_cast<int>(g < p.total_blocks ? g : p.total_blocks);
  const auto k = p.bf16 ? reduce_mean_kernel<true> : reduce_mean_kernel<false>;
  return launch_pdl(k, dim3(grid), dim3(kEltThreads), 0, s, p);
}

cudaError_t launch_replicate(const ReplParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0 || p.nrep <= 0) return cudaSuccess;
  const long long g = static_cast<long long>(sms) * 4;
  const int rgrid = static_cast<int>(g < p.total_blocks ? g : p.total_blocks);
  return launch_pdl(replicate_kernel, dim3(rgrid), dim3(kEltThreads), 0, s, p);
}

cudaError_t launch_schedule_advance(DevSched* s, long long total, double wu, double wd, double fin,
                                    cudaStream_t st) {
  return launch_pdl(schedule_advance_kernel, dim3(1), dim3(32), 0, st, s, total, wu, wd, fin);
}

// step <- step + 1; lr_mult <- linear climb over `warm` steps, then a cosine
// from 1 to final_frac at the last step, total - 1 ("Muon vs AdamW, Lion and
// Sophia: a fair race", the bake-off's schedule by step).
__global__ void schedule_cosine_kernel(DevSched* s, long long total, long long warm, double final_frac) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const long long step = s->step;  // 0-based index of the step being taken
  const long long last = total - 1;
  double m;
  if (step < warm) {
    m = static_cast<double>(step) / static_cast<double>(warm);
  } else if (step >= last || last <= warm) {
    m = final_frac;
  } else {
    const double phase = 3.141592653589793 * static_cast<double>(step - warm) / static_cast<double>(last - warm);
    m = final_frac + (1.0 - final_frac) * 0.5 * (1.0 + cos(phase));
  }
  s->step = step + 1;
  s->lr_mult = static_cast<float>(m);
}

cudaError_t launch_schedule_cosine(DevSched* s, long long total, long long warm, double fin, cudaStream_t st) {
  return launch_pdl(schedule_cosine_kernel, dim3(1), dim3(32), 0, st, s, total, warm, fin);
}

// ------------------------------------------------------------- launchers
int elt_chunk() { return kEltChunk; }
int adam_chunk() { return kAdamChunk; }

// Persistent grid: every SM filled to its occupancy limit, never more blocks
// than chunks.
template <typename K>
static int persistent_grid(K kernel, int chunks, int sms) {
  static thread_local const void* last_kernel = nullptr;
  static thread_local int last_occ = 0;
  if (last_kernel != reinterpret_cast<const void*>(kernel)) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kEltThreads, 0) != cudaSuccess || occ < 1)
      occ = 1;
    last_kernel = reinterpret_cast<const void*>(kernel);
    last_occ = occ;
  }
  const long long g = static_cast<long long>(sms) * last_occ;
  return static_cast<int>(g < chunks ? g : chunks);
}

template <bool GBF16>
static cudaError_t launch_momentum_bulk_t(const EltParams& p, int sms, cudaStream_t s) {
  auto k = momentum_bulk_kernel<GBF16>;
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BulkCfg<GBF16>::SMEM);
  if (e != cudaSuccess) return e;
  // as many blocks as are resident at once (three per SM with bf16 grads,
  // two with the larger fp32 stages): every block stays until the end
  static int per_sm = 0;   // per instantiation; the same for every device of a node
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kEltThreads, BulkCfg<GBF16>::SMEM) != cudaSuccess || n < 1)
      n = 1;
    per_sm = n;
  }
  const int cap = per_sm * sms;
  const int grid = p.total_items < cap ? p.total_items : cap;
  return launch_pdl(k, dim3(grid), dim3(kEltThreads), BulkCfg<GBF16>::SMEM, s, p);
}

cudaError_t launch_momentum_bulk(const EltParams& p, int sms, cudaStream_t s) {
  if (p.total_items <= 0) return cudaSuccess;
  return p.grad_bf16 ? launch_momentum_bulk_t<true>(p, sms, s) : launch_momentum_bulk_t<false>(p, sms, s);
}

int bulk_chunks() { return kBulkChunks; }

cudaError_t launch_momentum_norm(const EltParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  const auto k = p.grad_bf16 ? momentum_norm_kernel<true> : momentum_norm_kernel<false>;
  return launch_pdl(k, dim3(persistent_grid(k, p.total_blocks, sms)), dim3(kEltThreads), 0, s, p);
}

int rowq_class(int cols, bool vec) {
  if (!vec) return 3;
  if (cols <= kRowEqWarpCols) return 0;
  if (cols <= kRowEqBlockCols) return 1;
  if (cols <= kRowEqSmemCols) return 2;
  return 3;
}

// Grid for a persistent row kernel: every SM filled to the occupancy the
// block's dynamic shared memory allows, never more blocks than work items.
template <typename K>
static int rowq_grid(K k, int items, size_t smem, int sms) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kEltThreads, smem) != cudaSuccess || occ < 1)
    occ = 1;
  const long long g = static_cast<long long>(sms) * occ;
  return static_cast<int>(g < items ? g : items);
}

// Classes 2 and 3 share momentum_rowq_kernel; its dynamic shared memory is
// sized for the longest on-chip row of the launch (none for class 3).
template <bool GBF16>
static cudaError_t launch_rowq(const EltParams& p, int cls, int sms, cudaStream_t s) {
  if (cls == 0) {
    auto k = rowq_warp_kernel<GBF16>;
    const int wpb = kEltThreads / 32;
    return launch_pdl(k, dim3(rowq_grid(k, (p.total_blocks + wpb - 1) / wpb, 0, sms)), dim3(kEltThreads), 0, s, p);
  }
  if (cls == 1) {
    auto k = rowq_block_kernel<GBF16>;
    return launch_pdl(k, dim3(rowq_grid(k, p.total_blocks, 0, sms)), dim3(kEltThreads), 0, s, p);
  }
  auto k = momentum_rowq_kernel<GBF16>;
  // the attribute is set once per device; concurrent callers may both set it
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowEqSmemCols * 4)) !=
        cudaSuccess)
      return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  int cols = 0;
  for (int i = 0; i < p.nmats; ++i)
    if (p.mats[i].vec && p.mats[i].cols <= kRowEqSmemCols && p.mats[i].cols > cols) cols = p.mats[i].cols;
  const size_t smem = static_cast<size_t>((cols + 3) / 4) * sizeof(float4);
  return launch_pdl(k, dim3(rowq_grid(k, p.total_blocks, smem, sms)), dim3(kEltThreads), smem, s, p);
}

cudaError_t launch_momentum_rowq(const EltParams& p, int cls, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  return p.grad_bf16 ? launch_rowq<true>(p, cls, sms, s) : launch_rowq<false>(p, cls, sms, s);
}

cudaError_t launch_normuon_update(const EltParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  const int wpb = kEltThreads / 32;
  const long long need = (static_cast<long long>(p.total_blocks) + wpb - 1) / wpb;
  const long long cap = static_cast<long long>(sms) * 8;
  const int ngrid = static_cast<int>(need < cap ? need : cap);
  return launch_pdl(normuon_update_kernel, dim3(ngrid), dim3(kEltThreads), 0, s, p);
}

cudaError_t launch_norm_finalize(const EltParams& p, cudaStream_t s) {
  if (p.nmats <= 0) return cudaSuccess;
  return launch_pdl(norm_finalize_kernel, dim3(p.nmats), dim3(kEltThreads), 0, s, p);
}

cudaError_t launch_update(const EltParams& p, bool emit, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  const auto k = emit ? update_kernel<true> : update_kernel<false>;
  return launch_pdl(k, dim3(persistent_grid(k, p.total_blocks, sms)), dim3(kEltThreads), 0, s, p);
}

template <bool GBF16>
static cudaError_t launch_adamw_bulk_t(const AdamParams& p, int sms, cudaStream_t s) {
  auto k = adamw_bulk_kernel<GBF16>;
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, AdamBulkCfg<GBF16>::SMEM);
  if (e != cudaSuccess) return e;
  static int per_sm = 0;   // resident blocks per SM, per instantiation
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kEltThreads, AdamBulkCfg<GBF16>::SMEM) != cudaSuccess ||
        n < 1)
      n = 1;
    per_sm = n;
  }
  const int cap = per_sm * sms;
  const int grid = p.total_blocks < cap ? p.total_blocks : cap;
  return launch_pdl(k, dim3(grid), dim3(kEltThreads), AdamBulkCfg<GBF16>::SMEM, s, p);
}

cudaError_t adamw_status_address(unsigned int** addr) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(addr), g_adamw_status);
}

cudaError_t launch_adamw_bulk(const AdamParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  return p.grad_bf16 ? launch_adamw_bulk_t<true>(p, sms, s) : launch_adamw_bulk_t<false>(p, sms, s);
}

cudaError_t launch_adamw(const AdamParams& p, int sms, cudaStream_t s) {
  if (p.total_blocks <= 0) return cudaSuccess;
  const auto k = p.grad_bf16 ? adamw_kernel<true> : adamw_kernel<false>;
  return launch_pdl(k, dim3(persistent_grid(k, p.total_blocks, sms)), dim3(kEltThreads), 0, s, p);
}

}  // namespace muon
