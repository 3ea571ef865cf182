// Query-tile attention kernel on tcgen05 tensor cores.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss
// Function": the compressed cache's attention output Y_hat and log-sum-exp
// l_hat are matched to the full cache's (Y, l) over the training queries.
//
// One CTA owns 128 training queries of one head-problem and streams the
// problem's keys in tiles of 64.  Every product keeps about 16 significant
// bits through a bf16 hi/lo split, with fp32 accumulation in tensor memory:
//   S = Q K^T     Q_hi K_hi + Q_hi K_lo + Q_lo K_hi   (Q in TMEM, K in smem)
//   online softmax, one thread per query row and warpgroup, lazy rescaling
//   O += P V      P_hi V_hi + P_hi V_lo + P_lo V_hi   (P in TMEM over S, V in smem)
// Two row warpgroups take alternate key tiles, each with its own running
// max / sum and its own O accumulator; the two are merged at the end by their
// log-sum-exp (the same identity that merges chunks of a cache).
// Tensor memory (512 columns): S/P buffers at 0 and 64 (tile parity), O of
// warpgroup g at 128 + g*D, Q hi/lo after them.
// Modes:
//   LOSS     keys K_c, values V_c: writes l_hat, Go = dL/dY_hat (bf16),
//            delta = Go . Y_hat - dL/dl_hat (with the rounded Go), loss partials
//   TARGETS  keys K_z, values V_z: writes Y (fp32 and bf16 hi/lo) and l
//   STATS    row log-sum-exp only
//   WRITE_A  given l_hat: writes A = exp(S - l_hat) as bf16 hi/lo
// Warp roles: warps 0-7 rows (warp w <-> TMEM lanes 32 (w % 4) ..), warp 8 TMA
// producer, warp 9 TMEM allocator and MMA issuer.
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int BM = 128;          // queries per CTA
constexpr int BN = 64;           // keys per tile
constexpr int NTHREADS = 320;
constexpr float kRescale = 8.f;  // lazy rescale threshold (log2 units)
constexpr float L2E = 1.4426950408889634f;

template <int D, int MODE>
struct Fwd {
  static constexpr int KD = D / 64;
  static constexpr bool PV = (MODE == FWD_LOSS || MODE == FWD_TARGETS);
  static constexpr int NS = 3;
  static constexpr int T_BYTES = BN * D * 2;  // one 64-row bf16 tile (hi or lo)
  static constexpr int NT = PV ? 4 : 2;       // K hi, K lo (, V hi, V lo)
  static constexpr int STAGE = NT * T_BYTES;
  static constexpr int BYTES = NS * STAGE;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = 128;            // O of warpgroup g at COL_O + g * D
  static constexpr uint32_t COL_Q = COL_O + 2 * D;  // Q hi at +0, Q lo at +D/2
};

struct FwdBars {
  uint64_t q_full;
  uint64_t kv_full[3], kv_empty[3];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint32_t tmem;
  int abort;
  float m2[2][BM], l[2][BM];  // per warpgroup running max (log2) and sum
  float part[2][BM][2];       // per warpgroup half-row sums: |Yh - Y|^2, Go . Yh
  float red[16];
};

__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int D, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap mKh, const __grid_constant__ CUtensorMap mKl,
               const __grid_constant__ CUtensorMap mVh, const __grid_constant__ CUtensorMap mVl,
               FwdArgs a) {
  using C = Fwd<D, MODE>;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ FwdBars bars;
  const int b = blockIdx.y;
  if (a.flt.skip(b)) return;
  const int64_t q_begin = a.q_off[b];
  const int nq = (int)(a.q_off[b + 1] - q_begin);
  const int q0 = blockIdx.x * BM;
  if (q0 >= nq) return;
  const int64_t k_begin = a.k_off[b];
  const int nk = (int)(a.k_off[b + 1] - k_begin);
  const int ntiles = (nk + BN - 1) / BN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars.q_full, 2 * BM);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], C::PV ? 1 : BM);
      mbar_init(&bars.p_full[i], BM);
    }
    mbar_init(&bars.o_done, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&bars.tmem, C::TMEM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&mKh);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % C::NS;
        if (j >= C::NS && !mbar_wait(&bars.kv_empty[st], ((j / C::NS) - 1) & 1, abort)) {
          *abort = 1;
          break;
        }
        issued = j + 1;
        unsigned char *base = sm + st * C::STAGE;
        const int krow = (int)(k_begin + j * BN);
        mbar_arrive_expect_tx(&bars.kv_full[st], C::STAGE);
        for (int r = 0; r < C::KD; ++r) {
          tma_load_2d(base + r * BN * 128, &mKh, &bars.kv_full[st], 64 * r, krow);
          tma_load_2d(base + C::T_BYTES + r * BN * 128, &mKl, &bars.kv_full[st], 64 * r, krow);
          if (C::PV) {
            tma_load_2d(base + 2 * C::T_BYTES + r * BN * 128, &mVh, &bars.kv_full[st], 64 * r, krow);
            tma_load_2d(base + 3 * C::T_BYTES + r * BN * 128, &mVl, &bars.kv_full[st], 64 * r, krow);
          }
        }
      }
      if (*abort)  // let issued copies land before shared memory is released
        for (int j = (issued > C::NS ? issued - C::NS : 0); j < issued; ++j)
          mbar_wait(&bars.kv_full[j % C::NS], (j / C::NS) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(BM, BN, false, false);
      const uint32_t id_pv = idesc_bf16(BM, D, false, true);
      const uint32_t tq_hi = tmem + C::COL_Q, tq_lo = tmem + C::COL_Q + D / 2;
      bool ok = mbar_wait(&bars.q_full, 0, abort);
      fence_after_sync();
      auto issue_pv = [&](int i) -> bool {
        const int pb = i & 1;
        if (!mbar_wait(&bars.p_full[pb], (i >> 1) & 1, abort)) return false;
        fence_after_sync();
        const uint64_t vh0 = sdesc(smem_u32(sm + (i % C::NS) * C::STAGE + 2 * C::T_BYTES),
                                   BN * 128, 1024);
        const uint64_t vl0 = sdesc_add(vh0, C::T_BYTES);
        const uint32_t tp = tmem + pb * BN;            // P hi at +0, P lo at +32 columns
        const uint32_t to = tmem + C::COL_O + pb * D;  // O of the tile's warpgroup
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t vh = sdesc_add(vh0, kk * 2048), vl = sdesc_add(vl0, kk * 2048);
          mma_bf16_ts(to, tp + kk * 8, vh, id_pv, (i > 1 || kk > 0) ? 1u : 0u);
          mma_bf16_ts(to, tp + kk * 8, vl, id_pv, 1u);
          mma_bf16_ts(to, tp + 32 + kk * 8, vh, id_pv, 1u);
        }
        mma_commit(&bars.kv_empty[i % C::NS]);
        mma_commit(&bars.s_free[pb]);
        return true;
      };
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % C::NS, sb = j & 1;
        if (!mbar_wait(&bars.kv_full[st], (j / C::NS) & 1, abort)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&bars.s_free[sb], ((j >> 1) - 1) & 1, abort)) { ok = false; break; }
        fence_after_sync();
        const uint64_t kh0 = sdesc(smem_u32(sm + st * C::STAGE), 16, 1024);
        const uint64_t kl0 = sdesc_add(kh0, C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_k = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          const uint64_t kh = sdesc_add(kh0, off_k), kl = sdesc_add(kl0, off_k);
          mma_bf16_ts(tmem + sb * BN, tq_hi + kk * 8, kh, id_s, kk > 0 ? 1u : 0u);
          mma_bf16_ts(tmem + sb * BN, tq_hi + kk * 8, kl, id_s, 1u);
          mma_bf16_ts(tmem + sb * BN, tq_lo + kk * 8, kh, id_s, 1u);
        }
        mma_commit(&bars.s_full[sb]);
        if (!C::PV) mma_commit(&bars.kv_empty[st]);
        if (C::PV && j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && C::PV && ntiles > 0) ok = issue_pv(ntiles - 1);
      mma_commit(&bars.o_done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.o_done, 0);  // every MMA of this CTA has completed
    }
  } else {
    // ------------------------------------------------------------ row warps
    const int wg = warp >> 2;  // warpgroup: tiles j with j % 2 == wg
    const int row = tid & (BM - 1);
    const int q = q0 + row;
    const bool valid = q < nq;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    {
      // this warpgroup's half of the query row (hi, lo) into tensor memory:
      // the A operand of S = Q K^T
      const uint4 *qh = reinterpret_cast<const uint4 *>(a.q_hi + (q_begin + q) * D);
      const uint4 *ql = reinterpret_cast<const uint4 *>(a.q_lo + (q_begin + q) * D);
#pragma unroll 1
      for (int c0 = wg * 32; c0 < D / 2; c0 += 64) {
        uint32_t vh[32], vl[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 h = valid ? qh[c0 / 4 + e] : make_uint4(0, 0, 0, 0);
          const uint4 l = valid ? ql[c0 / 4 + e] : make_uint4(0, 0, 0, 0);
          vh[4 * e] = h.x; vh[4 * e + 1] = h.y; vh[4 * e + 2] = h.z; vh[4 * e + 3] = h.w;
          vl[4 * e] = l.x; vl[4 * e + 1] = l.y; vl[4 * e + 2] = l.z; vl[4 * e + 3] = l.w;
        }
        tmem_st32u(tmem + lane_base + C::COL_Q + c0, vh);
        tmem_st32u(tmem + lane_base + C::COL_Q + D / 2 + c0, vl);
      }
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(&bars.q_full);
    }
    const float sl2 = a.scale * L2E;  // score scale in log2 units
    float lrow2 = 0.f;                // WRITE_A: the given lse in log2 units
    if (MODE == FWD_WRITE_A && valid) lrow2 = a.lse_in[q_begin + q] * L2E;
    float mref = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = wg; j < ntiles; j += 2) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (j >> 1) & 1, abort));
      if (!ok) break;
      fence_after_sync();
      float s[BN];
      tmem_ld32(tmem + lane_base + sb * BN, s);
      tmem_ld32(tmem + lane_base + sb * BN + 32, s + 32);
      const int kvalid = nk - j * BN;
      if (kvalid < BN) {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = (c < kvalid) ? s[c] : -INFINITY;
      }
      if (!C::PV) {
        fence_before_sync();
        mbar_arrive(&bars.s_free[sb]);
      }
      if (MODE == FWD_WRITE_A) {
        // A = exp2(s sl2 - lse2), split into bf16 hi / lo, into the padded A buffer
        const int64_t arow = a.a_pad_off[b] + q0 + row;
        uint4 *dh = reinterpret_cast<uint4 *>(a.a_hi + arow * a.ld_a + j * BN);
        uint4 *dl = reinterpret_cast<uint4 *>(a.a_lo + arow * a.ld_a + j * BN);
#pragma unroll
        for (int ch = 0; ch < BN / 8; ++ch) {
          uint32_t h[4], l[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = valid ? exp2f(fmaf(s[ch * 8 + 2 * e], sl2, -lrow2)) : 0.f;
            const float p1 = valid ? exp2f(fmaf(s[ch * 8 + 2 * e + 1], sl2, -lrow2)) : 0.f;
            split_pack(p0, p1, h[e], l[e]);
          }
          dh[ch] = make_uint4(h[0], h[1], h[2], h[3]);
          dl[ch] = make_uint4(l[0], l[1], l[2], l[3]);
        }
        continue;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) mt = fmaxf(mt, s[c]);
      mt *= sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt > mref + kRescale || mref == -INFINITY) {
        const float mnew = fmaxf(mt, mref);
        if (mref != -INFINITY) {
          alpha = exp2f(mref - mnew);
          rescale = true;
        }
        mref = mnew;
      }
      float ts = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        s[c] = exp2f(fmaf(s[c], sl2, -mref));
        ts += s[c];
      }
      lsum = lsum * alpha + ts;
      if (C::PV) {
        // P (hi, lo) over the S buffer: the A operand of O_wg += P V
        uint32_t ph[32], pl[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) split_pack(s[2 * c], s[2 * c + 1], ph[c], pl[c]);
        tmem_st32u(tmem + lane_base + sb * BN, ph);
        tmem_st32u(tmem + lane_base + sb * BN + 32, pl);
        if (__any_sync(0xffffffffu, rescale)) {
          // O_wg *= alpha.  Its last update, PV of tile j-2, was issued before S of
          // tile j, whose completion this warp has observed, so O_wg is settled.
          // The TMEM access is warp-wide: rows without a new max use alpha = 1.
          const uint32_t to = tmem + lane_base + C::COL_O + wg * D;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld32(to + c0, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(to + c0, o);
          }
        }
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(&bars.p_full[sb]);
      }
    }
    if (!ok) *abort = 1;
    // ------------------------------------------------------------ epilogue
    if (MODE != FWD_WRITE_A) {
      // merge the two warpgroups' statistics: m = max(m0, m1), l = sum l_g 2^(m_g - m)
      bars.m2[wg][row] = mref;
      bars.l[wg][row] = lsum;
      rows_sync();
      const float m0 = bars.m2[0][row], m1 = bars.m2[1][row];
      const float mm = fmaxf(m0, m1);
      const float e0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mm);
      const float e1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mm);
      const float ltot = bars.l[0][row] * e0 + bars.l[1][row] * e1;
      const float lse = (mm + log2f(ltot)) * 0.6931471805599453f;
      if (C::PV) {
        if (!mbar_wait(&bars.o_done, 0, abort)) *abort = 1;
        fence_after_sync();
      }
      const float inv = 1.f / ltot;
      const float w0 = e0 * inv, w1 = e1 * inv;  // weights of O_0 and O_1
      const bool has1 = ntiles > 1;              // O_1 holds data
      const float c_out = 2.f * a.w_out / ((float)nq * (float)D);
      const float c_lse = 2.f * a.w_lse / (float)nq;
      const int64_t grow = q_begin + q;
      float se = 0.f, gy = 0.f;
      if (C::PV) {
        // this warpgroup's half of the row's columns
#pragma unroll 1
        for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
          float o[32], o1[32];
          tmem_ld32(tmem + lane_base + C::COL_O + c0, o);
          tmem_ld32(tmem + lane_base + C::COL_O + D + c0, o1);
          if (!valid) continue;
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = o[e] * w0 + (has1 ? o1[e] * w1 : 0.f);
          if (MODE == FWD_TARGETS) {
            float4 *y4 = reinterpret_cast<float4 *>(a.y_out + grow * D + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              y4[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
            uint4 *yh = reinterpret_cast<uint4 *>(a.y_hi + grow * D + c0);
            uint4 *yl = reinterpret_cast<uint4 *>(a.y_lo + grow * D + c0);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t h[4], l[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                split_pack(o[ch * 8 + 2 * e], o[ch * 8 + 2 * e + 1], h[e], l[e]);
              yh[ch] = make_uint4(h[0], h[1], h[2], h[3]);
              yl[ch] = make_uint4(l[0], l[1], l[2], l[3]);
            }
          } else {
            const float4 *y4 = reinterpret_cast<const float4 *>(a.y_in + grow * D + c0);
            float ev[32];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 v = y4[e];
              ev[4 * e] = o[4 * e] - v.x;
              ev[4 * e + 1] = o[4 * e + 1] - v.y;
              ev[4 * e + 2] = o[4 * e + 2] - v.z;
              ev[4 * e + 3] = o[4 * e + 3] - v.w;
            }
            uint4 *g4 = reinterpret_cast<uint4 *>(a.go + grow * D + c0);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t h[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i0 = ch * 8 + 2 * e;
                // delta uses the bf16-rounded Go that the backward's dP product sees,
                // so the rounding of Go cancels exactly in dP - delta.
                h[e] = pack_bf16(c_out * ev[i0], c_out * ev[i0 + 1]);
                const float g0 = __uint_as_float(h[e] << 16);
                const float g1 = __uint_as_float(h[e] & 0xffff0000u);
                se = fmaf(ev[i0], ev[i0], se);
                se = fmaf(ev[i0 + 1], ev[i0 + 1], se);
                gy = fmaf(g0, o[i0], gy);
                gy = fmaf(g1, o[i0 + 1], gy);
              }
              g4[ch] = make_uint4(h[0], h[1], h[2], h[3]);
            }
          }
        }
      }
      if (MODE == FWD_LOSS) {
        bars.part[wg][row][0] = se;
        bars.part[wg][row][1] = gy;
        rows_sync();
        if (wg == 0) {
          float ls = 0.f;
          se = bars.part[0][row][0] + bars.part[1][row][0];
          gy = bars.part[0][row][1] + bars.part[1][row][1];
          if (valid) {
            const float el = lse - a.lse_in[grow];
            ls = el * el;
            a.lse_out[grow] = lse;
            a.delta[grow] = gy - c_lse * el;
          } else {
            se = 0.f;
          }
          // deterministic per-CTA partial sums of the two loss terms
          se = warp_sum(se);
          ls = warp_sum(ls);
          if (lane == 0) {
            bars.red[warp] = se;
            bars.red[4 + warp] = ls;
          }
        }
        rows_sync();
        if (tid == 0) {
          float *part = a.partials + ((int64_t)b * a.tiles_per_problem + blockIdx.x) * 2;
          part[0] = (bars.red[0] + bars.red[1]) + (bars.red[2] + bars.red[3]);
          part[1] = (bars.red[4] + bars.red[5]) + (bars.red[6] + bars.red[7]);
        }
      } else if (wg == 0 && valid) {  // TARGETS, STATS
        a.lse_out[grow] = lse;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

template <int D, int MODE>
int launch_fwd_tc(const FwdMaps &m, const FwdArgs &a, int max_tiles, int B, cudaStream_t st) {
  using C = Fwd<D, MODE>;
  static_assert(C::SMEM + sizeof(FwdBars) <= 232448, "shared memory");
  auto kern = k_attn_fwd<D, MODE>;
  KVS_CUDA_TRY(set_smem_once(kern, C::SMEM));
  kern<<<dim3(max_tiles, B), NTHREADS, C::SMEM, st>>>(m.kh, m.kl, m.vh, m.vl, a);
  KVS_LAUNCH_CHECK("k_attn_fwd");
  return KVS_OK;
}

template int launch_fwd_tc<64, FWD_LOSS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_LOSS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_TARGETS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_TARGETS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_STATS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_STATS>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_WRITE_A>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_WRITE_A>(const FwdMaps &, const FwdArgs &, int, int, cudaStream_t);

}  // namespace kvs
