// Arguments and launchers of the tcgen05 attention kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "kvs_internal.cuh"
#include "kvs_tc.cuh"

namespace kvs {

enum FwdMode : int { FWD_LOSS = 0, FWD_TARGETS = 1, FWD_STATS = 2, FWD_WRITE_A = 3 };
enum BwdMode : int { BWD_DK = 0, BWD_COLSUM = 1 };

// Rows of one key / value tile of the query-tile kernel (the TMA box height of
// its key and value maps).
constexpr int FWD_BN = 128;
// Queries of one tile of the key-tile kernel (the TMA box height of its query
// and Go maps).
constexpr int BWD_BQ = 64;
// Tiles one CTA takes in turn (its grid is ceil(tiles / items)): key tiles of the
// key-tile kernel and query tiles of the query-tile kernel, for a whole batch and
// for a sub-batch that shares the GPU with others.
constexpr int BWD_ITEMS = 2;
constexpr int FWD_ITEMS = 3;
constexpr int FWD_ITEMS_SHARED = 3;

// dL/dY_hat = c (Y_hat - Y), c = 2 w_out / (n_q d), is carried as fp16 scaled by
// sigma = 2^-round(log2 c) (so that it sits in fp16's normal range; 1 when c = 0):
// the loss forward writes Go = fp16(sigma c (Y_hat - Y)) and delta in the same
// scale, the key gradient divides dK by sigma.  Powers of two keep the scaling
// exact.
__device__ __forceinline__ float go_scale(int nq, int d, float w_out) {
  const float c = 2.f * w_out / ((float)nq * (float)d);
  return c > 0.f ? exp2f(-rintf(log2f(c))) : 1.f;
}

// Tensor maps of the bf16 operands (2-D, [rows, d], box 64 columns x FWD_BN rows).
struct FwdMaps {
  CUtensorMap kh, kl, vh, vl;
  CUtensorMap qh, ql;     // query tiles (box 64 columns x FWD_BN rows)
  CUtensorMap y;          // LOSS: targets, fp32 [sum_q, d], box 32 columns x FWD_BN rows
};

struct FwdArgs {
  const int64_t *q_off;   // [B+1] query rows
  const int64_t *k_off;   // [B+1] key rows (compress zone or compressed pairs)
  Filter flt;
  float scale;            // 1/sqrt(d)
  const __nv_bfloat16 *q_hi, *q_lo;  // [sum_q, d] query split (loaded into tensor memory)
  // LOSS
  const float *y_in;      // [sum_q, d] targets
  const float *lse_in;    // [sum_q] target lse (LOSS) or given row lse (WRITE_A)
  float *lse_out;         // [sum_q] row lse of these keys
  __nv_bfloat16 *go;      // [padded q, d] dL/dY_hat, fp16 bits scaled by go_scale
  float *delta;           // [sum_q] Go . Y_hat - dL/dl_hat, in the scale of Go
  float *partials;        // [B, tiles_per_problem, 2]
  int tiles_per_problem;
  float w_out, w_lse;     // loss weights (means over n_q d and n_q)
  // TARGETS
  float *y_out;           // [sum_q, d]
  __nv_bfloat16 *y_hi, *y_lo;
  // WRITE_A
  __nv_bfloat16 *a_hi, *a_lo;  // [sum padded q, ld_a]
  int64_t ld_a;
  const int64_t *a_pad_off;    // [B+1] padded query rows of q_hi/lo, go, y_hi/lo and the A buffer
  const int64_t *k_pad;        // [B+1] padded key / value rows of the bf16 key and value maps
  int *err;               // timeout flag
  long long wait;         // cycles a pipeline wait may spin (wait_limit())
};

struct BwdMaps {
  CUtensorMap kh, kl;     // key tile, box 64 columns x 128 rows
  CUtensorMap qh, ql, g;  // query / Go tiles, box 64 columns x BWD_BQ rows
};

struct BwdArgs {
  const int64_t *q_off;
  const int64_t *k_off;
  Filter flt;
  float scale;
  const float *lse;       // [sum_q] row lse used to form the probabilities
  const float *delta;     // [sum_q] (DK)
  const float *v32;       // [sum_k, d] values (DK; split into fp16 hi/lo in tensor memory)
  float w_out;            // output-term weight (DK: the scale of Go, go_scale)
  const int64_t *q_pad, *k_pad;      // [B+1] padded rows of the query / Go and key / value maps
  float *dk;              // [sum_k, d] (DK): dL/dK, or nsplit partial sums dk_stride apart
  float *imp;             // [sum_k] (COLSUM): column sums of probabilities
  int *err;
  long long wait;
  int nsplit;             // query tiles of a problem split over this many CTAs (COLSUM: 1)
  int64_t dk_stride;      // floats between the partial sums of two splits
};

struct GemmMaps {
  CUtensorMap ah, al, bh, bl;
};

struct GemmArgs3 {
  const int64_t *a_pad_off;  // [B+1] padded K (query) row offsets of both operands' buffers
  const int64_t *m_off;      // [B+1] M extents (keys)
  int n_fixed;               // N extent of A^T Y (d); unused by the Gram
  const int64_t *b_row_off;  // [B+1] K-row offsets of the B operand (Gram: = a_pad_off)
  float *c;                  // output rows at m_off[b], ld = ldc
  int64_t ldc;
  float diag;                // added on the diagonal (Gram: lambda)
  int b_col_shift;           // Gram: 0 ; R: 0 (B columns start at 0)
  int *err;
  long long wait;
};

template <int D, int MODE>
int launch_fwd_tc(const FwdMaps &m, const FwdArgs &a, int max_tiles, int items, int B,
                  cudaStream_t st);
template <int D, int MODE>
int launch_bwd_tc(const BwdMaps &m, const BwdArgs &a, int max_tiles, int items, int B,
                  cudaStream_t st);
// R = A^T Y (N = a.n_fixed = d) in 128 x d tiles (maps with 64-row boxes).
int launch_gemm3_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int B, cudaStream_t st);
// The Gram matrix A^T A + diag I in 256 x 256 tiles (maps with 32-row boxes).
int launch_gram2_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int B, cudaStream_t st);

// Trailing update of the blocked ridge Cholesky (64-column panels) on tensor
// cores.  The panel's factor columns L (rows below the diagonal block) and the
// forward-solved rows y of the diagonal block are held as tf32 hi / lo pairs,
// written by the panel and diagonal-block kernels:
//   P: [2 parities][hi, lo][sum_c][64]     P[par][h][c_off[b] + i][t] = L[i][j0 + t]
//   Y: [2 parities][hi, lo][B * d][64]     Y[par][h][b d + c][t] = y[j0 + t][c]
// with par = (j0 / 64) % 2, so that the next panel can be written while the
// current update still reads its own.
struct CholTcMaps {
  CUtensorMap p;  // fp32, box 32 columns x 128 rows
  CUtensorMap y;  // fp32, box 32 columns x d rows
};

struct CholTcArgs {
  float *G;              // [sum_c, ld] Gram matrix / factor (lower triangle)
  float *R;              // [sum_c, d] right-hand sides
  const int64_t *c_off;  // [B+1]
  const int *dead;       // [B] problems whose factorisation stopped
  int64_t ld;            // multiple of 4
  int64_t sum_c;
  int B, d;
  int *err;
  long long wait;
};

// The trailing lower triangle and right-hand-side rows from j0 + 128 (the next
// panel's column block takes its update in the diagonal-block and panel kernels).
// max_c: the longest problem (grid size).
int launch_chol_update_tc(const CholTcMaps &m, const CholTcArgs &a, int j0, int max_c,
                          cudaStream_t st);

// Host: a 2-D bf16 tensor map over [rows, cols] (row-major) with a
// [box_rows, 64]-element box and 128-byte swizzle.
int make_map_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows);
// The same for fp32 elements ([box_rows, 32]-element box).
int make_map_f32(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows);

}  // namespace kvs
