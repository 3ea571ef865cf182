// Trailing update of the blocked ridge Cholesky on tcgen05 tensor cores
// ("KVSculpt: KV Cache Compression as Distillation", section 2 "Value
// Optimization": values in closed form by ridge regression, here through the
// Cholesky factor of A^T A + lambda I).
//
// After panel j (columns j0 .. j0 + 63) is factored, the trailing lower
// triangle and the right-hand sides take the rank-64 update
//   G_ik -= L_i L_k^T        R_i -= L_i y_j
// with L_i the panel's factor rows and y_j the diagonal block's forward-solved
// rows.  Both operands are K-major (64 contraction columns, contiguous), so each
// output tile is a 128 x N x 64 product.  It runs as three tf32 products of
// hi / lo splits (x = hi + lo, hi = x with its low 13 mantissa bits cleared):
//   L_i L_k^T ~ hi_i hi_k^T + hi_i lo_k^T + lo_i hi_k^T
// which keeps about 21 significant bits per product, close to the fp32 FMA
// update it replaces.  The splits are written by the panel and diagonal-block
// kernels, so the update only moves tiles: TMA loads the four operand tiles
// (128 rows x 64 columns each, two 32-column boxes, 128-byte swizzle), one
// thread issues 24 MMAs into a 128-column TMEM accumulator, and four epilogue
// warps subtract it from the output tile, which they copy into shared memory
// while the operands load.  A CTA takes several tiles in turn (a grid stride):
// the next tile's operands load and its products run into the second of two
// TMEM accumulators while the epilogue of the current tile drains the first,
// so the per-tile setup, copy latency and epilogue overlap.
//
// Tiles (per problem of size k): 128 x 128 tiles (ti >= tj) of the trailing
// triangle from s = j0 + 128, then the right-hand-side rows from s in 128-row
// tiles (N = d).  The column block j0 + 64 .. j0 + 127 and its right-hand-side
// rows belong to the next panel, whose diagonal-block and panel kernels apply
// this update to them themselves (they run beside this kernel).
// Diagonal tiles are written whole: the factor's upper triangle is scratch.
// Rows and columns past a problem's k read other rows of the operand buffers
// and only ever reach outputs that are not stored.
#include <math.h>

#include <cmath>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int CM = 128;                 // output rows per tile
constexpr int CBOX = CM * 128;          // one 32-column fp32 box of 128 rows
constexpr int COPND = 2 * CBOX;         // one 128 x 64 operand
constexpr int CSP = 132;                // output-tile row stride in shared memory (floats)
constexpr int CSMEM = 4 * COPND + CM * CSP * 4 + 1024;  // A hi, A lo, B hi, B lo, output tile
constexpr int CTHREADS = 192;           // warps 0-3 epilogue, 4 producer, 5 MMA
constexpr int CACC = 128;               // TMEM columns of one accumulator (two in turn)
constexpr int CMAX_ITEMS = 16;          // most tiles one CTA takes
static_assert(CSMEM <= 227 * 1024, "shared memory");

// 16-byte asynchronous copy global -> shared; bytes past src_bytes are zero.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

struct CTile {
  int ra;    // first output row (problem-local)
  int cb;    // first output column (G) or 0 (R)
  int n;     // MMA N
  bool rhs;  // output R (B operand from the y splits) instead of G
};

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Tiles of the update after the panel at j0 for a problem of size k: the trailing
// triangle from s = j0 + 128 (the column block at j0 + 64 is the next panel's,
// updated by the next diagonal-block and panel kernels themselves), then the
// right-hand-side rows from s.
__host__ __device__ inline int update_tiles(int k, int j0) {
  const int n = k - j0 - 128;
  const int m = n > 0 ? ceil_div(n, CM) : 0;
  return m * (m + 1) / 2 + m;
}

__device__ bool tile_of(int t, int j0, int k, int d, CTile *o) {
  const int s = j0 + 128, n = k - s;
  if (n <= 0) return false;
  const int m = ceil_div(n, CM);
  const int ntri = m * (m + 1) / 2;
  if (t < ntri) {
    int r = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while (r * (r + 1) / 2 > t) --r;
    while ((r + 1) * (r + 2) / 2 <= t) ++r;
    *o = CTile{s + CM * r, s + CM * (t - r * (r + 1) / 2), CM, false};
    return true;
  }
  t -= ntri;
  if (t < m) {
    *o = CTile{s + CM * t, 0, d, true};
    return true;
  }
  return false;
}

// full: the current tile's operands landed; done[u]: the products into
// accumulator u completed (its operands are free again); acc_free[u]: the
// epilogue has read accumulator u; all_done: every product of the CTA completed.
struct CBars {
  uint64_t full, done[2], acc_free[2], all_done;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(CTHREADS, 1)
    k_chol_update_tc(const __grid_constant__ CUtensorMap mP, const __grid_constant__ CUtensorMap mY,
                     CholTcArgs a, int j0) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ CBars bars;
  const int b = blockIdx.y;
  if (a.dead[b]) return;
  const int64_t row0 = a.c_off[b];
  const int k = (int)(a.c_off[b + 1] - row0);
  CTile t0;
  if (!tile_of(blockIdx.x, j0, k, a.d, &t0)) return;
  // tile i of this CTA: blockIdx.x + i gridDim.x, while the problem has it
  auto tile_at = [&](int i, CTile *o) {
    return i < CMAX_ITEMS && tile_of(blockIdx.x + i * gridDim.x, j0, k, a.d, o);
  };
  const int par = (j0 / 64) & 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars.full, 1);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars.done[u], 1);
      mbar_init(&bars.acc_free[u], 4);  // one arrival per epilogue warp
    }
    mbar_init(&bars.all_done, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&bars.tmem, 2 * CACC);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      CTile t;
      for (int i = 0; tile_at(i, &t); ++i) {
        // the previous tile's products have read the operand buffers
        if (i > 0 && !mbar_wait(&bars.done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort, a.wait)) {
          *abort = 1;
          break;
        }
        if (*abort) break;
        const uint32_t bytes = 2 * COPND + (t.rhs ? 2 * 2 * a.d * 128 : 2 * COPND);
        mbar_arrive_expect_tx(&bars.full, bytes);
        for (int h = 0; h < 2; ++h) {
          const int pa = (int)((par * 2 + h) * a.sum_c + row0 + t.ra);
          const int pb = t.rhs ? (int)((par * 2 + h) * (int64_t)a.B * a.d + (int64_t)b * a.d)
                               : (int)((par * 2 + h) * a.sum_c + row0 + t.cb);
          for (int r = 0; r < 2; ++r) {
            tma_load_2d(sm + h * COPND + r * CBOX, &mP, &bars.full, 32 * r, pa);
            tma_load_2d(sm + (2 + h) * COPND + r * CBOX, t.rhs ? &mY : &mP, &bars.full, 32 * r,
                        pb);
          }
        }
        issued = i + 1;
      }
      // let the last issued copies land before shared memory is released (every
      // earlier tile's copies were waited for by the products that read them)
      if (*abort && issued) mbar_wait(&bars.full, (issued - 1) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      CTile t;
      for (int i = 0; tile_at(i, &t); ++i) {
        const int u = i & 1;
        if (!mbar_wait(&bars.full, i & 1, abort, a.wait) ||
            (i >= 2 && !mbar_wait(&bars.acc_free[u], ((i - 2) >> 1) & 1, abort, a.wait))) {
          ok = false;
          break;
        }
        fence_after_sync();
        const uint32_t id = idesc_tf32(CM, t.n);
        const uint32_t s = smem_u32(sm);
        const uint32_t acc = tmem + u * CACC;
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t ab = s + (pass == 2 ? COPND : 0);          // A hi, A hi, A lo
          const uint32_t bb = s + (pass == 1 ? 3 : 2) * COPND;      // B hi, B lo, B hi
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * CBOX + (kk & 3) * 32;
            mma_tf32(acc, sdesc(ab + off, 16, 1024), sdesc(bb + off, 16, 1024), id,
                     (pass > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bars.done[u]);
      }
      mma_commit(&bars.all_done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.all_done, 0);  // every MMA of this CTA has completed
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w owns output rows 32 w .. 32 w + 31 (its TMEM lanes).  The output tile
    // is copied into shared memory while the products run (lane l: columns
    // 4 l .. 4 l + 3 of each row), the accumulator is subtracted there row by row
    // (thread = row), and the rows go back with whole-row stores.  Each warp
    // touches only its own rows of the staging tile.
    float *gs = reinterpret_cast<float *>(sm + 4 * COPND);
    CTile t;
    for (int i = 0; tile_at(i, &t); ++i) {
      const int u = i & 1;
      const int nv = t.n / 4;  // active lanes
      const int ncol = t.rhs ? a.d : k;
      float *out = t.rhs ? a.R + row0 * a.d : a.G + row0 * a.ld;
      const int64_t ldo = t.rhs ? a.d : a.ld;
      const int gc = t.cb + 4 * lane;
      const int cmax = ncol - gc;  // valid columns from this lane's first
      for (int q = 0; q < 32; ++q) {
        const int r = 32 * warp + q, gr = t.ra + r;
        if (lane < nv && gr < k && cmax > 0)
          cp_async16(gs + r * CSP + 4 * lane, out + (int64_t)gr * ldo + gc, 4 * min(cmax, 4));
      }
      cp_async_commit_wait();
      const bool ok = mbar_wait(&bars.done[u], (i >> 1) & 1, abort, a.wait) && !*abort;
      if (!ok) {
        *abort = 1;
        break;
      }
      fence_after_sync();
      __syncwarp();
      float *grow = gs + (32 * warp + lane) * CSP;
      const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
      for (int c0 = 0; c0 < t.n; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + u * CACC + lane_base + c0, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float4 *p = reinterpret_cast<float4 *>(grow + c0 + 4 * e);
          const float4 x = *p;
          *p = make_float4(x.x - v[4 * e], x.y - v[4 * e + 1], x.z - v[4 * e + 2],
                           x.w - v[4 * e + 3]);
        }
      }
      // accumulator u is free for the tile after next
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_free[u]);
      for (int q = 0; q < 32; ++q) {
        const int r = 32 * warp + q, gr = t.ra + r;
        if (lane >= nv || gr >= k || cmax <= 0) continue;
        const float4 v = *reinterpret_cast<const float4 *>(gs + r * CSP + 4 * lane);
        float *p = out + (int64_t)gr * ldo + gc;
        if (cmax >= 4) {
          *reinterpret_cast<float4 *>(p) = v;
        } else {
          p[0] = v.x;
          if (cmax > 1) p[1] = v.y;
          if (cmax > 2) p[2] = v.z;
        }
      }
      __syncwarp();
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    fence_after_sync();
    tmem_dealloc(tmem, 2 * CACC);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

// Tiles per CTA: the count that minimises an estimate of the kernel's time,
// whole waves of CTAs (one per SM) times the CTA's time (about 4 us for its
// first tile, 3 us for each further one).
static int update_items(int tiles, int B) {
  const int nsm = sm_count();
  int best = 1;
  double bc = 1e30;
  for (int it = 1; it <= CMAX_ITEMS; ++it) {
    const int ctas = ceil_div(tiles, it) * B;
    const double cost = std::ceil((double)ctas / nsm) * (4.0 + 3.0 * (it - 1));
    if (cost < bc - 1e-9) {
      bc = cost;
      best = it;
    }
    if (ceil_div(tiles, it) == 1) break;
  }
  return best;
}

int launch_chol_update_tc(const CholTcMaps &m, const CholTcArgs &a, int j0, int max_c,
                          cudaStream_t st) {
  KVS_CUDA_TRY(set_smem_once(k_chol_update_tc, CSMEM));
  const int tiles = update_tiles(max_c, j0);  // the longest problem has the most tiles
  if (tiles <= 0) return KVS_OK;
  const int per = ceil_div(tiles, update_items(tiles, a.B));
  k_chol_update_tc<<<dim3(per, a.B), CTHREADS, CSMEM, st>>>(m.p, m.y, a, j0);
  KVS_LAUNCH_CHECK("k_chol_update_tc");
  return KVS_OK;
}

}  // namespace kvs
