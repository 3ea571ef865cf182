// Adam on the compressed keys: the ablation of the key optimiser ("KVSculpt: KV
// Cache Compression as Distillation", summary §4 "Optimizer Efficacy": Adam in
// place of L-BFGS leaves a much larger per-layer error).  One elementwise pass
// over the batch's sum_c x d key values in float4 vectors, grid-stride over the
// SMs; the gradient comes from kvs_loss_grad.
#include "kvs_internal.cuh"

namespace kvs {
namespace {

__device__ __forceinline__ void adam1(float g, float &m, float &v, float &x, float lr, float b1,
                                      float b2, float eps, float bc1, float bc2) {
  m = fmaf(b1, m, (1.f - b1) * g);
  v = fmaf(b2, v, (1.f - b2) * (g * g));
  x -= lr * (m / bc1) / (sqrtf(v / bc2) + eps);
}

__global__ void __launch_bounds__(256) k_adam(float4 *__restrict__ x, const float4 *__restrict__ g,
                                              float4 *__restrict__ m, float4 *__restrict__ v,
                                              int64_t n4, float lr, float b1, float b2, float eps,
                                              float bc1, float bc2) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 gg = g[i];
    float4 mm = m[i], vv = v[i], xx = x[i];
    adam1(gg.x, mm.x, vv.x, xx.x, lr, b1, b2, eps, bc1, bc2);
    adam1(gg.y, mm.y, vv.y, xx.y, lr, b1, b2, eps, bc1, bc2);
    adam1(gg.z, mm.z, vv.z, xx.z, lr, b1, b2, eps, bc1, bc2);
    adam1(gg.w, mm.w, vv.w, xx.w, lr, b1, b2, eps, bc1, bc2);
    m[i] = mm;
    v[i] = vv;
    x[i] = xx;
  }
}

}  // namespace

int launch_adam(float *Kc, const float *dKc, float *m, float *v, int64_t n, float lr, float b1,
                float b2, float eps, float bc1, float bc2, cudaStream_t st) {
  const int64_t n4 = n / 4;
  if (n4 == 0) return KVS_OK;
  const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 148 * 8);  // grid-stride beyond
  k_adam<<<blocks, 256, 0, st>>>(reinterpret_cast<float4 *>(Kc),
                                 reinterpret_cast<const float4 *>(dKc),
                                 reinterpret_cast<float4 *>(m), reinterpret_cast<float4 *>(v), n4,
                                 lr, b1, b2, eps, bc1, bc2);
  KVS_LAUNCH_CHECK("k_adam");
  return KVS_OK;
}

}  // namespace kvs
