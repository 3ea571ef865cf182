// Host orchestration of the attention contractions: targets and importance,
// loss forward, dK_c backward and the ridge normal equations, on the tcgen05
// kernels (kvs_attn_fwd.cu, kvs_attn_bwd.cu, kvs_gemm3.cu).
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss
// Function", "Value Optimization" and "Initialization".
//
// Operands enter the tensor cores as bf16 hi/lo pairs, every product taking
// three MMAs (hi.hi + hi.lo + lo.hi, about 16 significant bits) except
// dP = Go V^T, where Go is a single bf16 and delta is formed from the same
// rounded Go, so that its rounding cancels exactly in dP - delta.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <cstdio>
#include <atomic>
#include <mutex>
#include <unordered_map>

#include "kvs_attn_tc.cuh"

namespace kvs {

// ------------------------------------------------------------ tensor maps

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

namespace {
struct MapKey {
  const void *base;
  uint64_t rows, cols;
  uint32_t box_rows, box_cols, elem;
  bool operator==(const MapKey &o) const {
    return base == o.base && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           box_cols == o.box_cols && elem == o.elem;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey &k) const {
    return std::hash<const void *>()(k.base) ^ (k.rows * 0x9E3779B97F4A7C15ull) ^
           (k.cols << 20) ^ ((uint64_t)k.box_rows << 40) ^ ((uint64_t)k.box_cols << 52) ^
           ((uint64_t)k.elem << 60);
  }
};
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;  // encoded descriptors, reused

// 2-D map over a row-major [rows, cols] array of `elem`-byte elements, box
// [box_rows, box_cols] with 128 bytes per box row (128-byte swizzle).
int make_map_2d(CUtensorMap *m, CUtensorMapDataType type, uint32_t elem, const void *base,
                uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const uint32_t box_cols = 128 / elem;
  const MapKey key{base, rows, cols, box_rows, box_cols, elem};
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *m = it->second;
      return KVS_OK;
    }
  }
  auto fn = encode_fn();
  if (!fn) {
    set_driver_error(-1, "cuTensorMapEncodeTiled entry point");
    return KVS_ECUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, type, 2, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char where[160];
    snprintf(where, sizeof where, "cuTensorMapEncodeTiled (%llu x %llu, elem %u, box %u x %u, base %p)",
             (unsigned long long)rows, (unsigned long long)cols, elem, box_rows, box_cols, base);
    set_driver_error((int)r, where);
    return KVS_ECUDA;
  }
  std::lock_guard<std::mutex> lock(g_map_mu);
  if (g_maps.size() > 4096) g_maps.clear();
  g_maps.emplace(key, *m);
  return KVS_OK;
}
}  // namespace

int make_map_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, box_rows);
}

int make_map_f32(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows) {
  return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, rows, cols, box_rows);
}

// Multiprocessor count of the current device, cached per device (several host
// threads may ask at once: relaxed atomics, the value is the same for all).
int sm_count() {
  static std::atomic<int> n[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = n[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  n[dev].store(v, std::memory_order_relaxed);
  return v;
}

namespace {

// ------------------------------------------------------ elementwise helpers

// Problem b's rows x[off[b] ..] split into (hi, lo) at rows pad[b] .. of the padded
// operand buffers; the rows between its own count and the padded count are zero.
// Problems the filter leaves out keep their split.
__global__ void k_split_pad(const float *__restrict__ x, const int64_t *off, const int64_t *pad,
                            int d, __nv_bfloat16 *__restrict__ hi,
                            __nv_bfloat16 *__restrict__ lo, Filter flt) {
  const int b = blockIdx.y;
  if (flt.skip(b)) return;
  const int64_t v4 = (off[b + 1] - off[b]) * d / 4;  // d is a multiple of 4
  const int64_t n4 = (pad[b + 1] - pad[b]) * d / 4;
  const float4 *src = reinterpret_cast<const float4 *>(x + off[b] * d);
  uint2 *h = reinterpret_cast<uint2 *>(hi + pad[b] * d);
  uint2 *l = reinterpret_cast<uint2 *>(lo + pad[b] * d);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = i < v4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    uint32_t h0, h1, l0, l1;
    tc::split_pack(v.x, v.y, h0, l0);
    tc::split_pack(v.z, v.w, h1, l1);
    h[i] = make_uint2(h0, h1);
    l[i] = make_uint2(l0, l1);
  }
}

// x [rows by off] -> padded (hi, lo) by pad; max_rows: the largest padded count.
int split_pad(const float *x, const int64_t *off, const int64_t *pad, int64_t max_rows, int d,
              __nv_bfloat16 *hi, __nv_bfloat16 *lo, int B, cudaStream_t st,
              Filter flt = Filter{nullptr, 0, 0}) {
  const int64_t n4 = max_rows * d / 4;
  if (n4 == 0) return KVS_OK;
  const int per = (int)std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256,
                                                              std::max(1, 4096 / B)));
  k_split_pad<<<dim3(per, B), 256, 0, st>>>(x, off, pad, d, hi, lo, flt);
  KVS_LAUNCH_CHECK("k_split_pad");
  return KVS_OK;
}

// pad[b] = sum_{b' < b} round_up(n_b', 128) for the queries, zones and (when
// present) pairs of the batch.
__global__ void k_pad_offsets(const int64_t *q_off, const int64_t *z_off, const int64_t *c_off,
                              int B, int64_t *qp, int64_t *zp, int64_t *cp) {
  const int64_t *src[3] = {q_off, z_off, c_off};
  int64_t *dst[3] = {qp, zp, cp};
  const int k = threadIdx.x;
  if (k >= 3 || !src[k]) return;
  int64_t s = 0;
  dst[k][0] = 0;
  for (int b = 0; b < B; ++b) {
    s += (src[k][b + 1] - src[k][b] + 127) / 128 * 128;
    dst[k][b + 1] = s;
  }
}

int max_pad(int n) { return (n + 127) / 128 * 128; }

// loss[b] from the per-CTA partial sums of the loss forward (fixed order).
__global__ void k_loss_reduce(const float *partials, int tiles, const int64_t *q_off, int d,
                              float w_out, float w_lse, float *loss, float *parts, Filter flt,
                              int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B || flt.skip(b)) return;
  const int nq = (int)(q_off[b + 1] - q_off[b]);
  const int nt = (nq + 127) / 128;
  double so = 0.0, sl = 0.0;
  for (int t = 0; t < nt; ++t) {
    so += partials[((int64_t)b * tiles + t) * 2];
    sl += partials[((int64_t)b * tiles + t) * 2 + 1];
  }
  const double out = so / ((double)nq * d), ls = sl / (double)nq;
  loss[b] = (float)(w_out * out + w_lse * ls);
  if (parts) {
    parts[2 * b] = (float)out;
    parts[2 * b + 1] = (float)ls;
  }
}

int max_qtiles(const HostGeom &g) { return (g.max_q + 127) / 128; }

// Work items per CTA of the attention kernels.  A whole batch takes several
// query (key) tiles per CTA, so that each CTA's setup and epilogue overlap its next
// tile; the sub-batches of a partitioned solve, which run beside one another on
// the same SMs, take one tile per CTA (shorter CTAs interleave better: measured
// on the 56-problem cache, 360 against 363-372 ms per solve step).
int fwd_items(const Batch &Bt) { return Bt.share > 1 ? FWD_ITEMS_SHARED : FWD_ITEMS; }
int bwd_items(const Batch &Bt) { return Bt.share > 1 ? 1 : BWD_ITEMS; }

// Query splits of the key gradient: the largest key-tile CTA of the batch runs
// `items` key tiles over ceil(nqt / sp) query tiles each.  The split count
// minimises an estimate of the kernel's time: whole waves of CTAs times the
// CTA's time (2.3 us per query tile, 7.5 us of setup, copies and epilogue per
// CTA, 3 us more per further key tile), plus the reduction of sp partial sums
// (bytes_per_sum each, read and summed at 6 TB/s), with at least 8 query tiles
// per split.
int bwd_split(int ctas, int nqt_max, double bytes_per_sum, int items) {
  const int nsm = sm_count();
  int best = 1;
  double bc = 1e30;
  for (int sp = 1; sp <= 4; ++sp) {  // the workspace holds four partial sums
    if (sp > 1 && nqt_max / sp < 8) break;
    const int per = (nqt_max + sp - 1) / sp;
    const double waves = std::ceil((double)ctas * sp / nsm);
    double cost = waves * (2.3 * items * per + 7.5 + 3.0 * (items - 1));
    if (sp > 1) cost += (sp + 1) * bytes_per_sum / 6e6;  // us
    if (cost < bc - 1e-9) {
      bc = cost;
      best = sp;
    }
  }
  return best;
}

// dK = sum of the splits' partial sums, in split order, for the problems the
// filter selects.
__global__ void k_dk_reduce(const float *__restrict__ part, int ns, int64_t stride,
                            const int64_t *c_off, int d, Filter flt, float *__restrict__ dk) {
  const int b = blockIdx.y;
  if (flt.skip(b)) return;
  const int64_t o = c_off[b] * d / 4, n = c_off[b + 1] * d / 4 - o;
  const float4 *p4 = reinterpret_cast<const float4 *>(part);
  float4 *d4 = reinterpret_cast<float4 *>(dk);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = p4[o + e];
    for (int z = 1; z < ns; ++z) {
      const float4 v = p4[z * (stride / 4) + o + e];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    d4[o + e] = acc;
  }
}

template <int D>
int targets_d(const Batch &Bt, const float *Q, const float *Kz, const float *Vz, float *Y,
              float *lse, float *imp, const Work &w) {
  const HostGeom &g = Bt.g;
  int rc;
  const kvs_batch *bb = Bt.b;
  if ((rc = split_pad(Q, bb->q_off, w.a_pad_off, max_pad(g.max_q), D, w.qh, w.ql, g.B, Bt.st)) ||
      (rc = split_pad(Kz, bb->z_off, w.z_pad, max_pad(g.max_z), D, w.kh, w.kl, g.B, Bt.st)) ||
      (rc = split_pad(Vz, bb->z_off, w.z_pad, max_pad(g.max_z), D, w.vh, w.vl, g.B, Bt.st)))
    return rc;
  FwdMaps fm;
  if ((rc = make_map_bf16(&fm.kh, w.kh, g.sum_zpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.kl, w.kl, g.sum_zpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.vh, w.vh, g.sum_zpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.vl, w.vl, g.sum_zpad, D, FWD_BN)))
    return rc;
  if ((rc = make_map_bf16(&fm.qh, w.qh, g.sum_qpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.ql, w.ql, g.sum_qpad, D, FWD_BN)))
    return rc;
  FwdArgs a{};
  a.q_off = Bt.b->q_off;
  a.k_off = Bt.b->z_off;
  a.a_pad_off = w.a_pad_off;
  a.k_pad = w.z_pad;
  a.q_hi = w.qh;
  a.q_lo = w.ql;
  a.flt = Filter{nullptr, 0, 0};
  a.scale = 1.f / sqrtf((float)D);
  a.y_out = Y;
  a.y_hi = w.yh;
  a.y_lo = w.yl;
  a.lse_out = lse;
  a.err = w.err;
  a.wait = wait_limit();
  if ((rc = launch_fwd_tc<D, FWD_TARGETS>(fm, a, max_qtiles(g), fwd_items(Bt), g.B, Bt.st))) return rc;
  if (!imp) return KVS_OK;
  BwdMaps bm;
  if ((rc = make_map_bf16(&bm.kh, w.kh, g.sum_zpad, D, 128)) ||
      (rc = make_map_bf16(&bm.kl, w.kl, g.sum_zpad, D, 128)) ||
      (rc = make_map_bf16(&bm.qh, w.qh, g.sum_qpad, D, BWD_BQ)) ||
      (rc = make_map_bf16(&bm.ql, w.ql, g.sum_qpad, D, BWD_BQ)))
    return rc;
  bm.g = bm.qh;
  BwdArgs ba{};
  ba.q_off = Bt.b->q_off;
  ba.k_off = Bt.b->z_off;
  ba.q_pad = w.a_pad_off;
  ba.k_pad = w.z_pad;
  ba.flt = Filter{nullptr, 0, 0};
  ba.scale = a.scale;
  ba.lse = lse;
  ba.imp = imp;
  ba.err = w.err;
  ba.wait = wait_limit();
  ba.nsplit = 1;
  return launch_bwd_tc<D, BWD_COLSUM>(bm, ba, (g.max_z + 127) / 128, bwd_items(Bt), g.B, Bt.st);
}

// bf16 hi/lo copies of the keys and values of the compressed pairs.
template <int D>
int prep_pairs(const Batch &Bt, const float *Kc, const float *Vc, const Work &w,
               Filter kflt = Filter{nullptr, 0, 0}) {
  const HostGeom &g = Bt.g;
  int rc = split_pad(Kc, Bt.b->c_off, w.c_pad, max_pad(g.max_c), D, w.kh, w.kl, g.B, Bt.st, kflt);
  if (rc || !Vc) return rc;
  return split_pad(Vc, Bt.b->c_off, w.c_pad, max_pad(g.max_c), D, w.vh, w.vl, g.B, Bt.st);
}

template <int D>
int forward_d(const Batch &Bt, const float *Q, const float *Kc, const float *Vc, const float *Y,
              const float *lse, float w_out, float w_lse, float *loss, float *parts, Filter flt,
              bool q_ready, bool pairs_ready, bool reduce, const Work &w) {
  const HostGeom &g = Bt.g;
  int rc;
  if (!q_ready && (rc = split_pad(Q, Bt.b->q_off, w.a_pad_off, max_pad(g.max_q), D, w.qh, w.ql,
                                  g.B, Bt.st)))
    return rc;
  if (!pairs_ready && (rc = prep_pairs<D>(Bt, Kc, Vc, w))) return rc;
  FwdMaps fm;
  if ((rc = make_map_bf16(&fm.kh, w.kh, g.sum_cpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.kl, w.kl, g.sum_cpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.vh, w.vh, g.sum_cpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.vl, w.vl, g.sum_cpad, D, FWD_BN)))
    return rc;
  if ((rc = make_map_bf16(&fm.qh, w.qh, g.sum_qpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.ql, w.ql, g.sum_qpad, D, FWD_BN)) ||
      (rc = make_map_f32(&fm.y, Y, g.sum_q, D, FWD_BN)))
    return rc;
  FwdArgs a{};
  a.q_off = Bt.b->q_off;
  a.k_off = Bt.b->c_off;
  a.a_pad_off = w.a_pad_off;
  a.k_pad = w.c_pad;
  a.q_hi = w.qh;
  a.q_lo = w.ql;
  a.flt = flt;
  a.scale = 1.f / sqrtf((float)D);
  a.y_in = Y;
  a.lse_in = lse;
  a.lse_out = w.lse_h;
  a.go = w.go;
  a.delta = w.delta;
  a.partials = w.partials;
  a.tiles_per_problem = max_qtiles(g);
  a.w_out = w_out;
  a.w_lse = w_lse;
  a.err = w.err;
  a.wait = wait_limit();
  if ((rc = launch_fwd_tc<D, FWD_LOSS>(fm, a, max_qtiles(g), fwd_items(Bt), g.B, Bt.st))) return rc;
  if (!reduce) return KVS_OK;
  k_loss_reduce<<<(g.B + 127) / 128, 128, 0, Bt.st>>>(w.partials, max_qtiles(g), Bt.b->q_off, D,
                                                      w_out, w_lse, loss, parts, flt, g.B);
  KVS_LAUNCH_CHECK("k_loss_reduce");
  return KVS_OK;
}

template <int D>
int backward_d(const Batch &Bt, const float *Vc, float w_out, float *dKc, Filter flt,
               const Work &w) {
  const HostGeom &g = Bt.g;
  int rc;
  BwdMaps bm;
  if ((rc = make_map_bf16(&bm.kh, w.kh, g.sum_cpad, D, 128)) ||
      (rc = make_map_bf16(&bm.kl, w.kl, g.sum_cpad, D, 128)) ||
      (rc = make_map_bf16(&bm.qh, w.qh, g.sum_qpad, D, BWD_BQ)) ||
      (rc = make_map_bf16(&bm.ql, w.ql, g.sum_qpad, D, BWD_BQ)) ||
      (rc = make_map_bf16(&bm.g, w.go, g.sum_qpad, D, BWD_BQ)))
    return rc;
  BwdArgs ba{};
  ba.q_off = Bt.b->q_off;
  ba.k_off = Bt.b->c_off;
  ba.q_pad = w.a_pad_off;
  ba.k_pad = w.c_pad;
  ba.flt = flt;
  ba.scale = 1.f / sqrtf((float)D);
  ba.lse = w.lse_h;
  ba.delta = w.delta;
  ba.v32 = Vc;
  ba.w_out = w_out;
  ba.dk = dKc;
  ba.err = w.err;
  ba.wait = wait_limit();
  ba.nsplit = 1;
  const int ktiles = (g.max_c + 127) / 128;
  const int items = bwd_items(Bt);
  const int ns = bwd_split((ktiles + items - 1) / items * g.B, (g.max_q + 63) / 64,
                           (double)g.sum_c * D * 4, items);
  if (ns > 1) {
    // partial sums of ns query ranges, then their fixed-order sum
    ba.nsplit = ns;
    ba.dk = w.dkp;
    ba.dk_stride = g.sum_c * D;
  }
  if ((rc = launch_bwd_tc<D, BWD_DK>(bm, ba, ktiles, items, g.B, Bt.st))) return rc;
  if (ns == 1) return KVS_OK;
  k_dk_reduce<<<dim3(std::min<int64_t>(((int64_t)g.max_c * D / 4 + 255) / 256, 32), g.B), 256, 0,
                Bt.st>>>(w.dkp, ns, g.sum_c * D, Bt.b->c_off, D, flt, dKc);
  KVS_LAUNCH_CHECK("k_dk_reduce");
  return KVS_OK;
}

template <int D>
int fit_d(const Batch &Bt, const float *Q, const float *Kc, const float *Y, float lam, float *Vc,
          int32_t *status, bool q_ready, bool y_ready, Filter stats, const Work &w) {
  const HostGeom &g = Bt.g;
  int rc;
  const kvs_batch *bb = Bt.b;
  if (!q_ready && (rc = split_pad(Q, bb->q_off, w.a_pad_off, max_pad(g.max_q), D, w.qh, w.ql,
                                  g.B, Bt.st)))
    return rc;
  if (!y_ready && (rc = split_pad(Y, bb->q_off, w.a_pad_off, max_pad(g.max_q), D, w.yh, w.yl,
                                  g.B, Bt.st)))
    return rc;
  if ((rc = prep_pairs<D>(Bt, Kc, nullptr, w))) return rc;
  FwdMaps fm;
  if ((rc = make_map_bf16(&fm.kh, w.kh, g.sum_cpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.kl, w.kl, g.sum_cpad, D, FWD_BN)))
    return rc;
  if ((rc = make_map_bf16(&fm.qh, w.qh, g.sum_qpad, D, FWD_BN)) ||
      (rc = make_map_bf16(&fm.ql, w.ql, g.sum_qpad, D, FWD_BN)))
    return rc;
  fm.vh = fm.kh;
  fm.vl = fm.kl;
  FwdArgs a{};
  a.q_off = Bt.b->q_off;
  a.k_off = Bt.b->c_off;
  a.a_pad_off = w.a_pad_off;
  a.k_pad = w.c_pad;
  a.q_hi = w.qh;
  a.q_lo = w.ql;
  a.flt = stats;  // problems whose l_hat in the workspace is not that of Kc
  a.scale = 1.f / sqrtf((float)D);
  a.lse_out = w.lse_h;
  a.err = w.err;
  a.wait = wait_limit();
  if ((rc = launch_fwd_tc<D, FWD_STATS>(fm, a, max_qtiles(g), fwd_items(Bt), g.B, Bt.st))) return rc;
  a.flt = Filter{nullptr, 0, 0};
  a.lse_in = w.lse_h;
  a.a_hi = w.ahi;
  a.a_lo = w.alo;
  a.ld_a = g.ld_a;
  a.a_pad_off = w.a_pad_off;
  if ((rc = launch_fwd_tc<D, FWD_WRITE_A>(fm, a, max_qtiles(g), fwd_items(Bt), g.B, Bt.st))) return rc;
  GemmMaps gm;
  if ((rc = make_map_bf16(&gm.ah, w.ahi, g.sum_qpad, g.ld_a, 32)) ||
      (rc = make_map_bf16(&gm.al, w.alo, g.sum_qpad, g.ld_a, 32)))
    return rc;
  gm.bh = gm.ah;
  gm.bl = gm.al;
  GemmArgs3 ga{};
  ga.a_pad_off = w.a_pad_off;
  ga.m_off = Bt.b->c_off;
  ga.n_fixed = 0;
  ga.b_row_off = w.a_pad_off;
  ga.c = w.gram;
  ga.ldc = g.ld_g;
  ga.diag = lam;
  ga.err = w.err;
  ga.wait = wait_limit();
  const int tm = (g.max_c + 127) / 128;
  if ((rc = launch_gram2_tc(gm, ga, tm, g.B, Bt.st))) return rc;
  if ((rc = make_map_bf16(&gm.ah, w.ahi, g.sum_qpad, g.ld_a, 64)) ||
      (rc = make_map_bf16(&gm.al, w.alo, g.sum_qpad, g.ld_a, 64)) ||
      (rc = make_map_bf16(&gm.bh, w.yh, g.sum_qpad, D, 64)) ||
      (rc = make_map_bf16(&gm.bl, w.yl, g.sum_qpad, D, 64)))
    return rc;
  ga.n_fixed = D;
  ga.b_row_off = w.a_pad_off;  // Y at the padded query rows: zero rows past each problem
  ga.c = w.R;
  ga.ldc = D;
  ga.diag = 0.f;
  if ((rc = launch_gemm3_tc(gm, ga, tm, g.B, Bt.st))) return rc;
  return launch_chol_solve(Bt, Vc, status, w);
}

}  // namespace

int launch_pad_offsets(const Batch &Bt, const Work &w) {
  k_pad_offsets<<<1, 32, 0, Bt.st>>>(Bt.b->q_off, Bt.b->z_off, Bt.b->c_off, Bt.g.B, w.a_pad_off,
                                      w.z_pad, w.c_pad);
  KVS_LAUNCH_CHECK("k_pad_offsets");
  return KVS_OK;
}

int launch_targets(const Batch &Bt, const float *Q, const float *Kz, const float *Vz, float *Y,
                   float *lse, float *imp, const Work &w) {
  return Bt.g.d == 64 ? targets_d<64>(Bt, Q, Kz, Vz, Y, lse, imp, w)
                      : targets_d<128>(Bt, Q, Kz, Vz, Y, lse, imp, w);
}

int launch_forward(const Batch &Bt, const float *Q, const float *Kc, const float *Vc,
                   const float *Y, const float *lse, float w_out, float w_lse, float *loss,
                   float *parts, Filter flt, bool q_ready, const Work &w, bool pairs_ready,
                   bool reduce) {
  return Bt.g.d == 64 ? forward_d<64>(Bt, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, flt,
                                      q_ready, pairs_ready, reduce, w)
                      : forward_d<128>(Bt, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, flt,
                                       q_ready, pairs_ready, reduce, w);
}

int launch_split_pairs(const Batch &Bt, const float *Kc, const float *Vc, const Work &w,
                       Filter kflt) {
  return Bt.g.d == 64 ? prep_pairs<64>(Bt, Kc, Vc, w, kflt) : prep_pairs<128>(Bt, Kc, Vc, w, kflt);
}

int launch_backward(const Batch &Bt, const float *Vc, float w_out, float *dKc, Filter flt,
                    const Work &w) {
  return Bt.g.d == 64 ? backward_d<64>(Bt, Vc, w_out, dKc, flt, w)
                      : backward_d<128>(Bt, Vc, w_out, dKc, flt, w);
}

int launch_fit(const Batch &Bt, const float *Q, const float *Kc, const float *Y, float lam,
               float *Vc, int32_t *status, bool q_ready, bool y_ready, const Work &w,
               Filter stats) {
  return Bt.g.d == 64 ? fit_d<64>(Bt, Q, Kc, Y, lam, Vc, status, q_ready, y_ready, stats, w)
                      : fit_d<128>(Bt, Q, Kc, Y, lam, Vc, status, q_ready, y_ready, stats, w);
}

}  // namespace kvs
