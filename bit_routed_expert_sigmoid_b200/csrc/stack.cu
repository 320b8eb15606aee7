// Residual stream of a stack of Flint MoE layers: between two layers, the previous layer's output is
// added to the fp32 residual and the next layer's input is the weightless RMSNorm of the residual,
// rounded once to bf16 (the 47 routed blocks of the model: Aijuus/flint-w4exp, model summary;
// norm weight folded away, eps 1e-6).
#include "kernels.cuh"

namespace flint {

namespace {

constexpr int kNormThreads = 256;                 // x 8 columns = H

// One CTA per token: x[t] += y[t] (when y is given), then z[t] = bf16(x[t] / sqrt(mean(x[t]^2) + eps))
// (when z is given). The sum of squares is reduced in a fixed order (per thread, then the warp
// butterfly, then the warps in order), so the result does not depend on scheduling.
__global__ void __launch_bounds__(kNormThreads) residual_rmsnorm_kernel(float* __restrict__ x,
                                                                        const uint16_t* __restrict__ y, float eps,
                                                                        uint16_t* __restrict__ z) {
  __shared__ float wsum[kNormThreads / 32];
  const int t = blockIdx.x;
  const int c = threadIdx.x * 8;
  float* xr = x + static_cast<size_t>(t) * kH + c;
  float4 a = *reinterpret_cast<const float4*>(xr);
  float4 b = *reinterpret_cast<const float4*>(xr + 4);
  float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  if (y) {
    const uint4 yv = *reinterpret_cast<const uint4*>(y + static_cast<size_t>(t) * kH + c);
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] += bf16lo_to_f32(yw[j]);
      v[2 * j + 1] += bf16hi_to_f32(yw[j]);
    }
    *reinterpret_cast<float4*>(xr) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(xr + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
  if (!z) return;
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s = fmaf(v[j], v[j], s);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, m);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) wsum[warp] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) tot += wsum[w];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(kH) + eps);
  uint4 out;
  uint32_t* ou = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int j = 0; j < 4; ++j) ou[j] = pack_bf162(v[2 * j] * inv, v[2 * j + 1] * inv);
  *reinterpret_cast<uint4*>(z + static_cast<size_t>(t) * kH + c) = out;
}

}  // namespace

cudaError_t launch_residual_rmsnorm(float* x, const uint16_t* y, int T, float eps, uint16_t* z, cudaStream_t s) {
  static_assert(kH == kNormThreads * 8, "one CTA of 256 threads x 8 columns per token");
  residual_rmsnorm_kernel<<<T, kNormThreads, 0, s>>>(x, y, eps, z);
  return cudaGetLastError();
}

}  // namespace flint
