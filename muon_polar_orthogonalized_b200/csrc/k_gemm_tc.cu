// k_gemm_tc.cu -- the Newton-Schulz GEMMs on the 5th-generation tensor cores.
//
// One quintic iteration ("Chapter 4: The MuonAdamW Optimizer", Polar Express:
// Newton-Schulz Orthogonalization; "3.9 Optimizers", Muon: Orthogonalizing
// the Update) is three products:
//   gram  A = s^2 X X^T          symmetric: each tile row starts at its
//                                diagonal 256-block, and A is stored in upper
//                                form (256x256 blocks on and above the diagonal)
//   poly  B' = a I + b A + c A A symmetric likewise; A A = A A^T since A is
//                                symmetric, so both operands are rows of A;
//                                K blocks left of a row block's diagonal are
//                                read transposed from the stored upper form;
//                                the epilogue reads the A tile for b*A, adds
//                                a on the diagonal and keeps, per row, the
//                                ratio r_i = B'_ii / bf16(B'_ii) in fp32
//   axpy  X' = s r (B' X)        = s (a X + B X) with B''s diagonal exact:
//                                row i of the product scaled by r_i makes
//                                its diagonal term exact; wide matrices; tall
//                                ones (iterated as X^T) compute
//                                X' = s (X B') r (column scale) in parameter
//                                layout; B' is read like A above.  a X rides
//                                in the product; the epilogue only scales
//   axpy_update                  last iteration: U = bf16(X') feeds the
//                                cautious-decay update of W directly
// s is the Frobenius scale 1/(||m~||+1e-7), applied on the first iteration
// only (X0 is stored unscaled; bf16 rounding is scale-free up to exponent).
//
// Structure: persistent grouped kernel, one CTA per SM (CTA pairs by
// default), a TMA -> shared-memory ring, tcgen05.mma kind::f16 (bf16 in, fp32
// accumulate) issued by one thread into TMEM, and eight (fused update:
// twelve) epilogue warps that drain TMEM with tcgen05.ld.  Tiles: 256x256 on
// a CTA pair with two 256-column accumulators (one tile's epilogue overlaps
// the next tile's MMAs) and a 3-stage ring of K = 128; the Gram and plain B'X
// products use 256x512 pair tiles (two N=256 MMAs per K step into one
// 512-column accumulator, 4-stage ring of K = 64).  Where row lengths allow, each operand block of a
// stage is one TMA box of a chunked 4-D tensor map.
// Single-CTA mode: 128x256 tiles, 4-stage ring of K = 64.
//   warp 0: TMA producer        warp 1: MMA issuer (+ TMEM owner)
//   warps 2-9: epilogue (warp w reads TMEM lanes 32*(w%4) .. +31; two warps
//              per lane quadrant split the tile's columns); the fused
//              update has warps 2-13, three per quadrant
// No TMA or bulk load uses multicast; the only multicast is the
// tcgen05.commit that signals an mbarrier in both CTAs of a pair.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "pdl.cuh"
#include "sm100.cuh"

namespace muon {

// Tile geometry.  Single-CTA mode: 128x256 tiles, one SM per tile.  Pair mode
// (cta_group::2): 256 x (256*NSUB) tiles on a CTA pair; each CTA stages 128
// rows of A and, per 256-column sub-tile, 128 rows (half) of B; the leader
// issues NSUB 256x256x16 MMAs per K step that read both CTAs' shared memory,
// and each CTA's TMEM holds its 128 accumulator rows.  NSUB = 1: two
// accumulators of 256 columns, so one tile's epilogue overlaps the next
// tile's MMAs.  NSUB = 2: one 512-column accumulator (all of TMEM), 25% fewer
// operand bytes per FLOP from L2, the epilogue drain no longer overlapped.
#ifndef MUON_TC_PAIR_STAGES
#define MUON_TC_PAIR_STAGES 3
#endif
#ifndef MUON_TC_NARROW_BK
#define MUON_TC_NARROW_BK 128
#endif
#ifndef MUON_TC_WIDE_STAGES
#define MUON_TC_WIDE_STAGES 4
#endif
#ifndef MUON_TC_RASTER_GN
#define MUON_TC_RASTER_GN 8
#endif

#ifndef MUON_TC_EPI_WARPS
#define MUON_TC_EPI_WARPS 8
#endif
#ifndef MUON_TC_UPD_EPI_WARPS
#define MUON_TC_UPD_EPI_WARPS 12
#endif
#ifndef MUON_TC_POLY_EPI_WARPS
#define MUON_TC_POLY_EPI_WARPS 8
#endif
// Output staging for the TMA row stores: per epilogue warp two 2 KB buffers of
// 32 rows x 32 bf16 (64-byte swizzle), used alternately.
constexpr int TC_STAGE_TILE_BYTES = 32 * 32 * 2;
// Epilogue warps: a multiple of 4, since warp w may only read TMEM lanes
// 32*(w%4) .. +31; the warps of a lane quadrant split the tile's 32-column
// chunks between them.  Eight by default (two per quadrant).  The fused
// update's epilogue (W read, masked, written per element) is the longer one:
// where K is short it outlasts the next tile's MMAs, so it gets twelve (three
// per quadrant), which its registers and shared memory allow (it stores from
// registers and needs no staging).
template <int EPI, int NSUB>
struct EpiCfg {
  static constexpr int WARPS = (EPI == EPI_AXPY_UPDATE && NSUB == 1) ? MUON_TC_UPD_EPI_WARPS
                               : (EPI == EPI_POLY && NSUB == 1)      ? MUON_TC_POLY_EPI_WARPS
                                                                     : MUON_TC_EPI_WARPS;
  static constexpr int SPLIT = WARPS / 4;                    // warps per lane quadrant
  static constexpr int THREADS = 64 + 32 * WARPS;            // producer + MMA + epilogue warps
  static constexpr bool STAGED = (EPI == EPI_GRAM || EPI == EPI_AXPY);   // rows leave by TMA stores
  static constexpr int STAGING_BYTES = STAGED ? WARPS * 2 * TC_STAGE_TILE_BYTES : 0;
  static constexpr int NCH = 256 * NSUB / 32;                // 32-column chunks per tile row
  static constexpr int MAX_CH = (NCH + SPLIT - 1) / SPLIT;   // most chunks one warp takes
  static_assert(WARPS % 4 == 0 && WARPS >= 4 && WARPS <= 16, "epilogue warps");
};
template <bool PAIR, int NSUB>
struct TcCfg {
  static_assert(NSUB == 1 || (PAIR && NSUB == 2), "512-column tiles need CTA pairs");
  static constexpr int BM = PAIR ? 256 : 128;        // tile rows
  static constexpr int BN = 256 * NSUB;              // tile columns
  // K per pipeline stage: 128 on 256x256 pair tiles (64 KB stages), else 64.
  // An SM's TMA ingest is set by the number of copies per stage more than by
  // their bytes (measured: a 32 KB stage moves 44 B/clk as two 16 KB boxes and
  // 57 B/clk as one 32 KB box; a 64 KB stage 78 B/clk as two 32 KB boxes),
  // and a 256x256 pair tile consumes 64 B/clk at the full MMA rate.
  static constexpr int BK = (PAIR && NSUB == 1) ? MUON_TC_NARROW_BK : 64;
  static constexpr int KCH = BK / 64;                // 64-wide K chunks per stage
  static constexpr int MN_CHUNK_BYTES = BK * 128;    // MN-major: one 64-wide MN chunk of BK k-rows
  static constexpr int A_ROWS = 128;                 // A rows staged per CTA
  static constexpr int SUB_B_ROWS = PAIR ? 128 : 256;  // B rows staged per CTA per 256-column sub-tile
  static constexpr int B_ROWS = SUB_B_ROWS * NSUB;
  static constexpr int A_CHUNK_BYTES = A_ROWS * 128;          // K-major: one 64-wide K chunk
  static constexpr int SUB_B_CHUNK_BYTES = SUB_B_ROWS * 128;
  static constexpr int A_BYTES = A_ROWS * BK * 2;
  static constexpr int SUB_B_BYTES = SUB_B_ROWS * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = NSUB == 2 ? MUON_TC_WIDE_STAGES : PAIR ? MUON_TC_PAIR_STAGES : 4;
  static_assert(BK == 64 || BK == 128, "K per stage");
  static_assert(kSymBlock % BK == 0, "a K block lies inside one 256-block of an upper-form operand");
  static constexpr int ACC_BUFS = NSUB == 1 ? 2 : 1;   // TMEM accumulators (512 columns in all)
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;          // barriers, TMEM slot, abort flag
  static constexpr int STAGING_OFF = BAR_OFF + 1024;            // output staging (EpiCfg::STAGING_BYTES)
  template <int EPI>
  static constexpr int smem_bytes() { return STAGING_OFF + EpiCfg<EPI, NSUB>::STAGING_BYTES + 1024 /*align slack*/; }
};
constexpr int TC_BN = 256;   // columns of one MMA (N) and of a narrow tile
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_RASTER_GN = MUON_TC_RASTER_GN;   // tile-column band width of the non-symmetric raster

struct TileCoord {
  int prob, mat, tm;
  int col0;   // first output column of the tile
};

// Columns one MMA of a tile computes: 256, or 128 for a 256-column tile
// (one sub-tile) of which at most 128 columns lie inside N (the ragged last
// tile column of a width that is an odd multiple of 128, e.g. 1664).  Such a
// tile runs N = 128 MMAs, half the work; with CTA pairs each CTA then stages
// 64 rows of B, so the second CTA's B rows start 64 (not 128) past col0.
template <int NSUB>
__device__ __forceinline__ int mma_cols(const GemmProblem& q, const TileCoord& tc) {
  return (NSUB == 1 && q.N - tc.col0 <= TC_BN / 2) ? TC_BN / 2 : TC_BN;
}

// A symmetric output's row block I (BM rows) starts its tiles at the
// 256-block of its rows on the diagonal: the upper form stores nothing left
// of it, so no tile computes a block that lies wholly below the diagonal.
template <int BM>
__host__ __device__ constexpr int sym_col_start(int I) {
  return kSymBlock * ((I * BM) / kSymBlock);
}

// Linear tile index -> (problem, matrix, tile row, first column).  Symmetric
// problems enumerate, per tile row I, the tiles from its diagonal 256-block
// rightwards (sym_col_start; the last one may reach past N, and its
// 256-column sub-tiles that lie wholly past N are neither loaded nor
// multiplied).  A column-major problem walks every tile row
// of one tile column before the next column (B'X of a wide matrix: the
// concurrent tiles share few X panels and all of B', which stays in L2, so
// each operand is read from DRAM about once); the others walk bands of
// TC_RASTER_GN tile columns row by row.
template <int BM, int BN>
__device__ __forceinline__ TileCoord decode_tile(const TcGemmParams& p, int t) {
  int pi = 0;
  while (pi + 1 < p.nprob && t >= p.prob[pi + 1].tile_begin) ++pi;
  const GemmProblem& q = p.prob[pi];
  int lt = t - q.tile_begin;
  const int mat = lt / q.tiles_per_mat;
  int r = lt - mat * q.tiles_per_mat;
  int tm, tn;
  if (q.sym) {
    int I = 0;
    for (;;) {
      const int c0 = sym_col_start<BM>(I);
      const int cnt = (q.N - c0 + BN - 1) / BN;
      if (r < cnt) break;
      r -= cnt;
      ++I;
    }
    return {pi, mat, I, sym_col_start<BM>(I) + r * BN};
  } else if (q.col_major) {
    tn = r / q.tiles_m;
    tm = r - tn * q.tiles_m;
  } else {
    const int band_tiles = q.tiles_m * TC_RASTER_GN;
    const int band = r / band_tiles;
    const int rem = r - band * band_tiles;
    const int width = min(TC_RASTER_GN, q.tiles_n - band * TC_RASTER_GN);
    tm = rem / width;
    tn = band * TC_RASTER_GN + (rem - (rem / width) * width);
  }
  return {pi, mat, tm, tn * BN};
}

__device__ __forceinline__ void record_timeout(unsigned int* status, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(status, kDevTimeout);
}

// Row store of one chunk straight from registers (A*A products): 2 x 32
// bytes per lane where the row is 32-byte aligned, else 4 x 16 bytes.
__device__ __forceinline__ void st_bf16x32(__nv_bfloat16* dst, const float (&v)[32], bool v8) {
  uint4 d[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      __nv_bfloat162 b = __floats2bfloat162_rn(v[q * 8 + h * 2], v[q * 8 + h * 2 + 1]);
      w[h] = *reinterpret_cast<uint32_t*>(&b);
    }
    d[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (v8) {
    sm100::st_global_v8(dst, d[0], d[1]);
    sm100::st_global_v8(dst + 16, d[2], d[3]);
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d4[q] = d[q];
  }
}

// The Gram and B'X epilogues instead stage their rows for a TMA store (the
// staged store measured faster there; for A*A the direct store was faster).
// One warp's 32 rows x 32 columns of output, lane = row: packed to bf16 into a
// 2 KB staging buffer in the 64-byte-swizzle layout (16-byte unit u of row r
// at unit u ^ ((r >> 1) & 3), four shared-memory wavefronts per store), then
// written by one TMA store at (j0, y, mat).  The buffer used two chunks ago
// is reused once its store has finished reading it.  Rows >= M and columns
// >= N of the box are clipped by the tensor map; a box that starts at or
// beyond row M is not issued.  Warp-uniform; every lane calls it.
__device__ __forceinline__ void stage_row_store(const CUtensorMap* tmap, uint8_t* buf, int lane,
                                                const float (&v)[32], int j0, int y, int M, int mat) {
  if (lane == 0) sm100::bulk_wait_group_read<1>();
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      __nv_bfloat162 b = __floats2bfloat162_rn(v[u * 8 + h * 2], v[u * 8 + h * 2 + 1]);
      w[h] = *reinterpret_cast<uint32_t*>(&b);
    }
    const int su = u ^ ((lane >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + lane * 64 + su * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  sm100::fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && y < M) {
    sm100::tma_store_3d(tmap, buf, j0, y, mat);
    sm100::bulk_commit_group();
  }
}

// The same update for two neighbouring elements, with packed fp32 arithmetic
// (fma.rn.f32x2: per lane the same rounding as fmaf, so the same bits).  The
// mask drops cautious_w's w == 0 test: where w = +-0, wd*w + u is u for any
// u != 0, and u == 0 keeps the mask on anyway, so the result is unchanged.
// u0, u1: bf16(v0), bf16(v1) from one packed conversion.
__device__ __forceinline__ float2 cautious_w2(float2 w, float v0, float v1, float lr, float wd, bool cautious) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(v0, v1);
  const uint32_t bits = *reinterpret_cast<const uint32_t*>(&b);
  const float2 u = make_float2(__uint_as_float(bits << 16), __uint_as_float(bits & 0xffff0000u));
  const float2 t = __ffma2_rn(make_float2(wd, wd), w, u);   // decayed
  float2 tm = t;
  if (cautious) {
    // decay off where the signs differ and u != 0
    const bool off0 = ((__float_as_int(u.x) ^ __float_as_int(w.x)) < 0) && (u.x != 0.f);
    const bool off1 = ((__float_as_int(u.y) ^ __float_as_int(w.y)) < 0) && (u.y != 0.f);
    tm.x = off0 ? u.x : t.x;
    tm.y = off1 ? u.y : t.y;
  }
  return __ffma2_rn(make_float2(-lr, -lr), tm, w);
}

__device__ __forceinline__ float cautious_w(float w, float u, float lr, float wd, bool cautious) {
  bool mask = true;
  if (cautious) {
    const bool sdiff = (__float_as_uint(u) ^ __float_as_uint(w)) >> 31;
    mask = !sdiff || u == 0.f || w == 0.f;
  }
  const float t = mask ? fmaf(wd, w, u) : u;
  return fmaf(-lr, t, w);
}

// ------------------------------------------------------------- epilogue
// Each epilogue thread owns one accumulator row i of the tile and walks it in
// 32-column chunks.  Per chunk: (1) issue the global loads the epilogue needs
// (the b*A / a*X operand, and W for the fused update) as independent loads,
// (2) read the accumulator chunk from TMEM, (3) combine and store.  Before
// waiting for a tile's accumulator, the thread prefetches its row segments of
// those operands into L2, so the loads in (1) hit L2.

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

template <int EPI>
__device__ __forceinline__ void epilogue_prefetch(const TcGemmParams& p, const GemmProblem& q,
                                                  int mat, int i, int jt, int width) {
  if (EPI == EPI_GRAM || EPI == EPI_AXPY || i >= q.M) return;
  const int ncols = min(width, q.N - jt);  // jt < N
  if (EPI == EPI_POLY) {
    const char* ein = reinterpret_cast<const char*>(
        static_cast<const __nv_bfloat16*>(q.ein) + mat * q.ein_bs + static_cast<long long>(i) * q.ein_ld + jt);
    for (int b = 0; b < ncols * 2; b += 128) prefetch_l2(ein + b);
  }
  if (EPI == EPI_AXPY_UPDATE) {
    const int wi = q.w_first + mat;
    const char* w = reinterpret_cast<const char*>(p.wptr[wi] + static_cast<long long>(i) * p.wcols[wi] + jt);
    for (int b = 0; b < ncols * 4; b += 128) prefetch_l2(w + b);
  }
}

struct EpiIn {
  uint4 e[4];     // 32 bf16 of the epilogue operand A (A*A products)
};
struct EpiW {
  float4 w[8];    // 32 fp32 parameters (fused update)
};

// The bf16 operand A of one chunk (A*A products only).
template <int EPI>
__device__ __forceinline__ void epilogue_load(const TcGemmParams& p, const GemmProblem& q, int mat,
                                              int i, int j0, bool full, EpiIn& in) {
  if (i >= q.M) return;
  if (EPI == EPI_POLY && full) {
    const __nv_bfloat16* src =
        static_cast<const __nv_bfloat16*>(q.ein) + mat * q.ein_bs + static_cast<long long>(i) * q.ein_ld + j0;
    if (((q.ein_ld | q.ein_bs) & 15) == 0) {   // 32-byte rows (the buffers are 1024-byte aligned)
      sm100::ld_global_v8(src, in.e[0], in.e[1]);
      sm100::ld_global_v8(src + 16, in.e[2], in.e[3]);
    } else {
      const uint4* e4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
      for (int k = 0; k < 4; ++k) in.e[k] = e4[k];
    }
  }
}

// The parameters W of one chunk (fused update).
template <int EPI>
__device__ __forceinline__ void epilogue_load_w(const TcGemmParams& p, const GemmProblem& q, int mat,
                                                int i, int j0, bool full, bool wvec, EpiW& in) {
  if (i >= q.M) return;
  if (EPI == EPI_AXPY_UPDATE && full && wvec) {
    const int wi = q.w_first + mat;
    const float* src = p.wptr[wi] + static_cast<long long>(i) * p.wcols[wi] + j0;
    if ((reinterpret_cast<uintptr_t>(src) & 31u) == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        sm100::ld_global_v8(src + 8 * k, *reinterpret_cast<uint4*>(&in.w[2 * k]),
                            *reinterpret_cast<uint4*>(&in.w[2 * k + 1]));
    } else {
      const float4* w4 = reinterpret_cast<const float4*>(src);
#pragma unroll
      for (int k = 0; k < 8; ++k) in.w[k] = w4[k];
    }
  }
}

__device__ __forceinline__ void unpack_bf16x32(const uint4 (&e)[4], float (&a)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {e[q].x, e[q].y, e[q].z, e[q].w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
      a[q * 8 + h * 2] = f.x;
      a[q * 8 + h * 2 + 1] = f.y;
    }
  }
}

// Called by every lane of the warp (the tall B'X column scale is shuffled).
// dsc: B'X's diagonal scale r of this thread's row (wide), or of column
// j0 + lane (tall: lane c supplies column j0 + c's to every lane).
template <int EPI>
__device__ __forceinline__ void epilogue_store(const TcGemmParams& p, const GemmProblem& q, int mat,
                                               int i, int j0, bool full, bool wvec,
                                               const EpiIn& in, const EpiW& win, float dsc,
                                               float (&v)[32]) {
  float f = 1.f;
  if (q.scale_mode) {
    const float s = p.scales[q.scale_base + mat];
    f = (q.scale_mode == 1) ? s * s : s;
  }
  if constexpr (EPI == EPI_AXPY || EPI == EPI_AXPY_UPDATE) {
    // both orientations multiply the accumulator by the one product r * s,
    // so that a matrix and its transpose give the same bits
    if (q.dsc) {
      if (q.dsc_col) {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] *= __shfl_sync(0xffffffffu, dsc, c) * f;
        f = 1.f;
      } else {
        f *= dsc;
      }
    }
  }
  if (i >= q.M) return;
  if constexpr (EPI == EPI_POLY) {
    float a[32];
    if (full) {
      unpack_bf16x32(in.e, a);
    } else {
      const __nv_bfloat16* ein = static_cast<const __nv_bfloat16*>(q.ein) + mat * q.ein_bs +
                                 static_cast<long long>(i) * q.ein_ld + j0;
#pragma unroll
      for (int c = 0; c < 32; ++c) a[c] = (j0 + c < q.N) ? __bfloat162float(ein[c]) : 0.f;
    }
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = fmaf(q.cb, a[c], q.cc * v[c]) + ((j0 + c == i) ? q.ca : 0.f);
    if (q.dsc && i >= j0 && i < j0 + 32) {
      // this row's diagonal element d: keep d / bf16(d), by which B'X scales
      // the product's row i so that its diagonal term d X_i comes out exact
      float d = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (j0 + c == i) d = v[c];
      const float h = __bfloat162float(__float2bfloat16_rn(d));
      q.dsc[mat * q.dsc_bs + i] = (h != 0.f) ? d / h : 1.f;
    }
  } else {
    // Gram: s^2 on the first iteration; axpy: s on the first iteration
    // (packed: the same product per element)
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const float2 r = __fmul2_rn(make_float2(v[c], v[c + 1]), make_float2(f, f));
      v[c] = r.x;
      v[c + 1] = r.y;
    }
  }

  if constexpr (EPI == EPI_AXPY_UPDATE) {
    // W and each of its copies (rptr: the other ranks' replicas, possibly in
    // peer GPUs' memory) receive the same new values, with plain stores
    const int wi = q.w_first + mat;
    const long long roff = static_cast<long long>(i) * p.wcols[wi] + j0;
    float* w = p.wptr[wi] + roff;
    const bool cautious = p.cautious != 0;
    const float lr = p.sched ? q.lr * p.sched->lr_mult : q.lr;
    if (full && wvec) {
      float4 nw[8];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 ww = win.w[c4];
        const float2 lo = cautious_w2(make_float2(ww.x, ww.y), v[c4 * 4 + 0], v[c4 * 4 + 1], lr, p.wd, cautious);
        const float2 hi = cautious_w2(make_float2(ww.z, ww.w), v[c4 * 4 + 2], v[c4 * 4 + 3], lr, p.wd, cautious);
        nw[c4] = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      // W and each copy: 32-byte stores where the row segment is 32-byte aligned
      auto store_row = [&](float* dst) {
        if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            sm100::st_global_v8(dst + 8 * k, *reinterpret_cast<const uint4*>(&nw[2 * k]),
                                *reinterpret_cast<const uint4*>(&nw[2 * k + 1]));
        } else {
          float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) d4[c4] = nw[c4];
        }
      };
      store_row(w);
      for (int r = 0; r < p.nrep; ++r) store_row(p.rptr[r][wi] + roff);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (j0 + c < q.N) {
          const float nv = cautious_w(w[c], __bfloat162float(__float2bfloat16_rn(v[c])), lr, p.wd, cautious);
          w[c] = nv;
          for (int r = 0; r < p.nrep; ++r) p.rptr[r][wi][roff + c] = nv;
        }
    }
  } else if constexpr (EPI == EPI_POLY) {
    __nv_bfloat16* row = static_cast<__nv_bfloat16*>(q.out) + mat * q.out_bs + static_cast<long long>(i) * q.out_ld + j0;
    if (full) {
      st_bf16x32(row, v, ((q.out_ld | q.out_bs) & 15) == 0);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (j0 + c < q.N) row[c] = __float2bfloat16_rn(v[c]);
    }
  }
  // Gram and B'X: the row goes out through stage_row_store
}

template <int EPI, bool PAIR, int NSUB>
__global__ void __launch_bounds__(EpiCfg<EPI, NSUB>::THREADS, 1)
tc_gemm_kernel(const __grid_constant__ TcGemmParams p) {
  using C = TcCfg<PAIR, NSUB>;
  using E = EpiCfg<EPI, NSUB>;
  static_assert(C::template smem_bytes<EPI>() <= 232448, "shared memory per block");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty_bar = full_bar + C::STAGES;
  uint64_t* tfull_bar = empty_bar + C::STAGES;   // [2]
  uint64_t* tempty_bar = tfull_bar + 2;          // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* staging = smem + C::STAGING_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = PAIR ? static_cast<int>(sm100::cluster_ctarank()) : 0;
  const int unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;        // tile-processing unit
  const int nunits = PAIR ? (gridDim.x >> 1) : gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      sm100::mbar_init(&full_bar[s], 1);
      sm100::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&tfull_bar[b], 1);
      sm100::mbar_init(&tempty_bar[b], (PAIR ? 2 : 1) * E::WARPS);   // one arrival per epilogue warp
    }
    *abort_flag = 0;
    sm100::fence_mbar_init();
    for (int i = 0; i < p.nprob; ++i) {
      sm100::prefetch_tmap(&p.tmA[i]);
      sm100::prefetch_tmap(&p.tmB[i]);
    }
  }
  if (warp == 1) {
    if (PAIR) {
      sm100::tmem_alloc_pair(tmem_slot, TC_TMEM_COLS);
      sm100::tmem_relinquish_pair();
    } else {
      sm100::tmem_alloc(tmem_slot, TC_TMEM_COLS);
      sm100::tmem_relinquish();
    }
  }
  sm100::tc_fence_before();
  __syncwarp();
  if (PAIR) sm100::cluster_sync(); else __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above touched only this CTA's shared memory, TMEM and the
  // kernel parameters; from here on global memory is read and written
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase_mask = 0;  // per stage: loads issued / their phase
      bool ok = true;
      for (int t = unit; t < p.total_tiles && ok; t += nunits) {
        const TileCoord tc = decode_tile<C::BM, C::BN>(p, t);
        const GemmProblem& q = p.prob[tc.prob];
        const int kblocks = (q.K + C::BK - 1) / C::BK;
        const int arow = tc.tm * C::BM + rank * C::A_ROWS;
        // B rows this CTA stages (sub-tile n adds n * TC_BN): half of the
        // MMA's columns per CTA of a pair
        const int brow = tc.col0 + rank * (C::SUB_B_ROWS * mma_cols<NSUB>(q, tc) / TC_BN);
        // 256-column sub-tiles wholly past N are neither loaded nor multiplied
        const int nact = min(NSUB, (q.N - tc.col0 + TC_BN - 1) / TC_BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!sm100::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
            record_timeout(p.status, abort_flag);
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          if (!PAIR || rank == 0)
            sm100::mbar_arrive_expect_tx(&full_bar[stage], (PAIR ? 2 : 1) * (C::A_BYTES + nact * C::SUB_B_BYTES));
          issued_mask |= 1u << stage;
          issued_phase_mask = (issued_phase_mask & ~(1u << stage)) | (phase << stage);
          const int k0 = kb * C::BK;
          const uint32_t leader_full = PAIR ? sm100::mapa_shared(sm100::smem_u32(&full_bar[stage]), 0) : 0;
          auto load = [&](uint8_t* dst, const CUtensorMap* m, int x, int y) {
            if (PAIR) sm100::tma_load_3d_pair(dst, m, leader_full, x, y, tc.mat);
            else sm100::tma_load_3d(dst, m, &full_bar[stage], x, y, tc.mat);
          };
          auto load4 = [&](uint8_t* dst, const CUtensorMap* m, int y, int z) {
            if (PAIR) sm100::tma_load_4d_pair(dst, m, leader_full, 0, y, z, tc.mat);
            else sm100::tma_load_4d(dst, m, &full_bar[stage], 0, y, z, tc.mat);
          };
          // `rows` operand rows from row0 for this K block.  Shared-memory
          // layout: K-major [K chunk][row][64 k]; MN-major [MN chunk][BK k][64 mn].
          // Chunked maps bring it in one box; otherwise one box per 64-wide chunk.
          auto load_operand = [&](uint8_t* dst, const CUtensorMap* m, bool mn, int row0, int rows) {
            if (q.chunked) {
              if (mn) load4(dst, m, k0, row0 / 64);
              else load4(dst, m, row0, k0 / 64);
            } else if (mn) {
              for (int h = 0; h < rows / 64; ++h) load(dst + h * C::MN_CHUNK_BYTES, m, row0 + h * 64, k0);
            } else {
#pragma unroll
              for (int c = 0; c < C::KCH; ++c) load(dst + c * rows * 128, m, k0 + c * 64, row0);
            }
          };
          // an upper-form operand's K block left of its rows' diagonal block
          // comes transposed from the block above the diagonal (MN-major)
          const bool a_t = q.a_sym && (k0 / kSymBlock) < (arow / kSymBlock);
          load_operand(sa, a_t ? &p.tmA2[tc.prob] : &p.tmA[tc.prob], q.a_mn || a_t, arow, C::A_ROWS);
#pragma unroll
          for (int n = 0; n < NSUB; ++n) {
            if (n >= nact) break;
            const int brow_n = brow + n * TC_BN;
            const bool b_t = q.b_sym && (k0 / kSymBlock) < (brow_n / kSymBlock);
            load_operand(sb + n * C::SUB_B_BYTES, b_t ? &p.tmB2[tc.prob] : &p.tmB[tc.prob], q.b_mn || b_t,
                         brow_n, C::SUB_B_ROWS);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && (!PAIR || rank == 0)) {
        // drain: let every load issued into this CTA's barriers land before exit
        for (int s = 0; s < C::STAGES; ++s) {
          if (!((issued_mask >> s) & 1u)) continue;
          const uint64_t t0 = sm100::globaltimer();
          while (!sm100::mbar_try_wait(&full_bar[s], (issued_phase_mask >> s) & 1u) &&
                 sm100::globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && (!PAIR || rank == 0)) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = unit; t < p.total_tiles && ok; t += nunits) {
        const TileCoord tc = decode_tile<C::BM, C::BN>(p, t);
        const GemmProblem& q = p.prob[tc.prob];
        const int kblocks = (q.K + C::BK - 1) / C::BK;
        // 256-row blocks of the operand rows (the same for both CTAs of a pair)
        const int ablk = (tc.tm * C::BM) / kSymBlock;
        const int bblk0 = tc.col0 / kSymBlock;
        const int nact = min(NSUB, (q.N - tc.col0 + TC_BN - 1) / TC_BN);   // sub-tiles reaching N
        if (!sm100::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) {
          record_timeout(p.status, abort_flag);
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!sm100::mbar_wait(&full_bar[stage], phase, abort_flag)) {
            record_timeout(p.status, abort_flag);
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          // descriptors of this K block, built once: the single issuing thread
          // must keep up with MMAs of ~128 cycles, so the inner loop only adds
          // the K16 offset to the start-address field ((address >> 4) in 14
          // bits; stage offsets never carry out of it)
          const uint32_t sa = sm100::smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
          const int kblk = (kb * C::BK) / kSymBlock;
          const bool a_mn = q.a_mn || (q.a_sym && kblk < ablk);
          const uint64_t ad0 = a_mn ? sm100::make_sdesc(sa, C::MN_CHUNK_BYTES, 1024) : sm100::make_sdesc(sa, 16, 1024);
          uint64_t bd0[NSUB];
          bool bmn[NSUB];
          uint32_t idn[NSUB];
#pragma unroll
          for (int n = 0; n < NSUB; ++n) {
            bmn[n] = q.b_mn || (q.b_sym && kblk < bblk0 + (n * TC_BN) / kSymBlock);
            const uint32_t sbn = sb + n * C::SUB_B_BYTES;
            bd0[n] = bmn[n] ? sm100::make_sdesc(sbn, C::MN_CHUNK_BYTES, 1024) : sm100::make_sdesc(sbn, 16, 1024);
            idn[n] = sm100::make_idesc_bf16(C::BM, mma_cols<NSUB>(q, tc), a_mn ? 1 : 0, bmn[n] ? 1 : 0);
          }
          // start-address step (16-byte units) of K16 step kk: MN-major 2048 B
          // per step; K-major 32 B per step within a 64-wide chunk, then the
          // next chunk
          auto koff = [](bool mn, int kk, int chunk_bytes) -> uint64_t {
            return mn ? static_cast<uint64_t>(kk * (2048 >> 4))
                      : static_cast<uint64_t>(((kk >> 2) * chunk_bytes + (kk & 3) * 32) >> 4);
          };
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
#pragma unroll
            for (int n = 0; n < NSUB; ++n) {
              if (n >= nact) break;
              const uint64_t ad = ad0 + koff(a_mn, kk, C::A_CHUNK_BYTES);
              const uint64_t bd = bd0[n] + koff(bmn[n], kk, C::SUB_B_CHUNK_BYTES);
              const uint32_t dn = d_tmem + static_cast<uint32_t>(n * TC_BN);
              if (PAIR) sm100::umma_bf16_pair(dn, ad, bd, idn[n], (kb | kk) ? 1u : 0u);
              else sm100::umma_bf16(dn, ad, bd, idn[n], (kb | kk) ? 1u : 0u);
            }
          }
          if (PAIR) sm100::umma_commit_pair_both(&empty_bar[stage]);
          else sm100::umma_commit(&empty_bar[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR) sm100::umma_commit_pair_both(&tfull_bar[acc]);
        else sm100::umma_commit(&tfull_bar[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;                          // TMEM lane quadrant this warp may read
    const int slice = (warp - 2) / 4;                   // which column slice of the tile
    constexpr int kChunks = E::MAX_CH;                  // 32-column chunks per warp, at most
    const int ch0 = slice * E::NCH / E::SPLIT;          // this warp's chunks: [ch0, ch0 + nch)
    const int nch = (slice + 1) * E::NCH / E::SPLIT - ch0;
    const int row_in_cta = quad * 32 + lane;
    uint8_t* my_staging = staging + (warp - 2) * 2 * TC_STAGE_TILE_BYTES;   // used when E::STAGED
    int stage_ctr = 0;   // staging buffer in use: stage_ctr & 1
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = unit; t < p.total_tiles; t += nunits) {
      const TileCoord tc = decode_tile<C::BM, C::BN>(p, t);
      const GemmProblem& q = p.prob[tc.prob];
      const int row0 = tc.tm * C::BM + rank * 128;   // first row this CTA holds
      const int i = row0 + row_in_cta;
      const int jslice = tc.col0 + ch0 * 32;
      if (jslice < q.N) epilogue_prefetch<EPI>(p, q, tc.mat, i, jslice, nch * 32);
      bool wvec = true;
      if (EPI == EPI_AXPY_UPDATE && i < q.M) {
        const int wi = q.w_first + tc.mat;
        wvec = ((reinterpret_cast<uintptr_t>(p.wptr[wi]) | (static_cast<uintptr_t>(p.wcols[wi]) << 2)) & 15u) == 0;
      }
      // Active chunks form one range [c_lo, c_hi): a symmetric tile skips the
      // chunks left of its rows' 256-block (a prefix) and a ragged tile stops
      // at N.  A*A loads its operand A one chunk ahead (the first one before
      // the accumulator is ready); the fused update loads W (prefetched to L2
      // above) with each chunk; the Gram and B'X epilogues load nothing but
      // B'X's diagonal scales, once per tile.  (Requesting chunk c+1's
      // accumulator columns from TMEM before storing chunk c measured no
      // faster on the wide products.)
      // symmetric output in upper form: chunks left of the rows' 256-block are not stored
      const int rblk = row0 / kSymBlock;
      int c_hi = 0;
      if (jslice < q.N) c_hi = min(nch, (q.N - jslice + 31) / 32);
      int c_lo = 0;
      if (q.sym) c_lo = max(0, (kSymBlock * rblk - jslice) / 32);
      auto chunk_j0 = [&](int cc) { return jslice + cc * 32; };
      constexpr bool kOperand = (EPI == EPI_POLY);   // operand loaded one chunk ahead
      auto load_operand = [&](int cc, EpiIn& in) {
        if constexpr (kOperand) epilogue_load<EPI>(p, q, tc.mat, i, chunk_j0(cc), chunk_j0(cc) + 32 <= q.N, in);
      };
      EpiIn ea, eb;   // operands of the even / odd chunk of a pair
      if (c_lo < c_hi) load_operand(c_lo, ea);
      // B'X: r_i of this thread's row (wide), or r_j of column jslice + 32 u
      // + lane for each chunk u (tall; shuffled to every lane in the epilogue)
      float dsc_row = 1.f;
      float dsc_t[kChunks];
#pragma unroll
      for (int u = 0; u < kChunks; ++u) dsc_t[u] = 1.f;
      if constexpr (EPI == EPI_AXPY || EPI == EPI_AXPY_UPDATE) {
        if (q.dsc) {
          const float* d = q.dsc + tc.mat * q.dsc_bs;
          if (!q.dsc_col) {
            if (i < q.M) dsc_row = d[i];
          } else {
#pragma unroll
            for (int u = 0; u < kChunks; ++u) {
              const int jc = jslice + u * 32 + lane;
              if (jc < q.N) dsc_t[u] = d[jc];
            }
          }
        }
      }
      auto dsc_of = [&](int cc) {   // selects, no indexed register array
        float r = dsc_row;
        if (q.dsc_col) {
          r = dsc_t[0];
#pragma unroll
          for (int u = 1; u < kChunks; ++u)
            if (cc == u) r = dsc_t[u];
        }
        return r;
      };
      if (!sm100::mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) {
        record_timeout(p.status, abort_flag);
        break;
      }
      sm100::tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * C::BN);
      auto tmem_req = [&](int cc, uint32_t (&r)[32]) {
        sm100::tmem_ld32_async(t_row + static_cast<uint32_t>((ch0 + cc) * 32), r);
      };
      auto process = [&](int cc, const EpiIn& in) {
        const int j0 = chunk_j0(cc);
        const bool full = (j0 + 32 <= q.N);
        EpiW win;
        epilogue_load_w<EPI>(p, q, tc.mat, i, j0, full, wvec, win);
        uint32_t r[32];
        tmem_req(cc, r);
        sm100::tmem_wait_ld(r);
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
        epilogue_store<EPI>(p, q, tc.mat, i, j0, full, wvec, in, win, dsc_of(cc), v);
        if constexpr (EPI == EPI_GRAM || EPI == EPI_AXPY) {
          stage_row_store(&p.tmOut[tc.prob], my_staging + (stage_ctr & 1) * TC_STAGE_TILE_BYTES, lane, v, j0,
                          row0 + quad * 32, q.M, tc.mat);
          ++stage_ctr;
        }
      };
      if constexpr (kOperand) {
#pragma unroll 1
        for (int cc = c_lo; cc < c_hi; cc += 2) {
          if (cc + 1 < c_hi) load_operand(cc + 1, eb);
          process(cc, ea);
          if (cc + 1 < c_hi) {
            if (cc + 2 < c_hi) load_operand(cc + 2, ea);
            process(cc + 1, eb);
          }
        }
      } else {
#pragma unroll 1
        for (int cc = c_lo; cc < c_hi; ++cc) process(cc, ea);
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_u32(&tempty_bar[acc]), 0));
        else sm100::mbar_arrive(&tempty_bar[acc]);
      }
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) sm100::bulk_wait_group<0>();   // every staged store written
  }

  sm100::tc_fence_before();
  __syncwarp();
  if (PAIR) sm100::cluster_sync(); else __syncthreads();
  sm100::tc_fence_after();
  // every role is done: the next kernel may be scheduled (triggering at the
  // start would let its blocks sit beside this CTA for the whole kernel,
  // e.g. AdamW's beside the fused update, and take issue slots from it)
  pdl_launch_dependents();
  if (warp == 1) {
    __syncwarp();
    if (PAIR) sm100::tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
    else sm100::tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

// ----------------------------------------------------------- self-test
// One thread waits on an mbarrier that nothing arrives on, with the bounded
// wait above and a short limit, and records the timeout in the status word.
__global__ void selftest_wait_kernel(unsigned int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  if (!sm100::mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicOr(status, kDevTimeout);
}

cudaError_t launch_selftest_wait(unsigned int* status, unsigned long long limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- launcher
int tc_tile_m(bool pair) { return pair ? TcCfg<true, 1>::BM : TcCfg<false, 1>::BM; }
int tc_tile_n(bool wide) { return wide ? TcCfg<true, 2>::BN : TC_BN; }
int tc_b_box_rows(bool pair) { return pair ? TcCfg<true, 1>::SUB_B_ROWS : TcCfg<false, 1>::SUB_B_ROWS; }
int tc_bk(bool pair, bool wide) {
  return wide ? TcCfg<true, 2>::BK : pair ? TcCfg<true, 1>::BK : TcCfg<false, 1>::BK;
}

template <int EPI, bool PAIR, int NSUB>
static cudaError_t launch_tc_epi(const TcGemmParams& p, int num_sms, cudaStream_t s) {
  using C = TcCfg<PAIR, NSUB>;
  constexpr int kSmem = C::template smem_bytes<EPI>();
  auto kern = tc_gemm_kernel<EPI, PAIR, NSUB>;
  static thread_local int max_units = 0;   // co-resident tile units (CTAs or CTA pairs)
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(EpiCfg<EPI, NSUB>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_units == 0) {
      cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1)
        clusters = num_sms / 2;
      max_units = clusters;
    }
  } else {
    max_units = num_sms;
  }
  const int units = p.total_tiles < max_units ? p.total_tiles : max_units;
  cfg.gridDim = dim3((PAIR ? 2 : 1) * units, 1, 1);
  // programmatic dependent launch (pdl.cuh): the kernel waits for the
  // previous grid before its first global-memory access
  attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs += 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_tc_gemm(const TcGemmParams& p, int epi, bool pair, bool wide, int num_sms, cudaStream_t s) {
  if (p.total_tiles <= 0) return cudaSuccess;
  if (wide && !pair) return cudaErrorInvalidValue;
  if (wide) {
    switch (epi) {
      case EPI_GRAM: return launch_tc_epi<EPI_GRAM, true, 2>(p, num_sms, s);
      case EPI_POLY: return launch_tc_epi<EPI_POLY, true, 2>(p, num_sms, s);
      case EPI_AXPY: return launch_tc_epi<EPI_AXPY, true, 2>(p, num_sms, s);
      case EPI_AXPY_UPDATE: return launch_tc_epi<EPI_AXPY_UPDATE, true, 2>(p, num_sms, s);
    }
  } else if (pair) {
    switch (epi) {
      case EPI_GRAM: return launch_tc_epi<EPI_GRAM, true, 1>(p, num_sms, s);
      case EPI_POLY: return launch_tc_epi<EPI_POLY, true, 1>(p, num_sms, s);
      case EPI_AXPY: return launch_tc_epi<EPI_AXPY, true, 1>(p, num_sms, s);
      case EPI_AXPY_UPDATE: return launch_tc_epi<EPI_AXPY_UPDATE, true, 1>(p, num_sms, s);
    }
  } else {
    switch (epi) {
      case EPI_GRAM: return launch_tc_epi<EPI_GRAM, false, 1>(p, num_sms, s);
      case EPI_POLY: return launch_tc_epi<EPI_POLY, false, 1>(p, num_sms, s);
      case EPI_AXPY: return launch_tc_epi<EPI_AXPY, false, 1>(p, num_sms, s);
      case EPI_AXPY_UPDATE: return launch_tc_epi<EPI_AXPY_UPDATE, false, 1>(p, num_sms, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace muon
