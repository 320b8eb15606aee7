// Weight preparation: bf16 expert weights -> the layer's int4 g128 (rotated) and NVFP4 formats.
// int4: Aijuus/flint-w4exp, summary table, weights row (codes i4, group 128, bf16 scale, fwht128
// rotation). NVFP4: kekzle/Flint-NVFP4, "What is in the files" (E2M1 codes, E4M3 scale per 16, F32
// tensor scale per Linear). The readings of the rounding rules are in include/flint_quant.h.
//
// These are HBM-bound streaming kernels (2 bytes read and about 0.53 written per weight). Every
// quantisation decision is taken in IEEE fp32 with one rounding per operation (the _rn intrinsics,
// so that the compiler cannot contract or approximate) and in a fixed order, which makes the codes
// independent of scheduling.
#include <cuda_runtime.h>
#include <stdint.h>

#include "flint_quant.h"

namespace flint {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint32_t kInvSqrt128Bits = 0x3DB504F3u;      // the fp32 nearest to 2^-3.5

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp32 -> bf16 bits, round to nearest even (finite values)
__device__ __forceinline__ uint32_t f32_to_bf16_rne(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// ---------------------------------------------------------------------------------------------
// int4 g128: a warp takes kGroupsPerWarp consecutive (row, 128-group) units, all of whose loads it
// issues before any arithmetic (HBM needs several KB in flight per SM); lane l holds elements
// 4l .. 4l+3 of a group.
constexpr int kGroupsPerWarp = 4;

__device__ __forceinline__ void quant_int4_group(float (&v)[4], int lane, bool rotate, uint32_t& sb_out,
                                                 uint32_t& packed) {
  if (rotate) {
    // Sylvester butterfly, stages h = 1, 2 (inside the lane) then 4 .. 64 (partner lane l ^ h/4):
    // the pair (i, i + h), i & h = 0, becomes (v_i + v_i+h, v_i - v_i+h)
    float a = v[0], b = v[1];
    v[0] = __fadd_rn(a, b);
    v[1] = __fsub_rn(a, b);
    a = v[2], b = v[3];
    v[2] = __fadd_rn(a, b);
    v[3] = __fsub_rn(a, b);
    a = v[0], b = v[2];
    v[0] = __fadd_rn(a, b);
    v[2] = __fsub_rn(a, b);
    a = v[1], b = v[3];
    v[1] = __fadd_rn(a, b);
    v[3] = __fsub_rn(a, b);
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float o = __shfl_xor_sync(kFull, v[j], m);
        v[j] = upper ? __fsub_rn(o, v[j]) : __fadd_rn(v[j], o);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = __fmul_rn(v[j], __uint_as_float(kInvSqrt128Bits));
  }
  float mx = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
  const uint32_t sb = f32_to_bf16_rne(__fdiv_rn(mx, 7.0f));
  const float s = __uint_as_float(sb << 16);
  const float rs = s > 0.f ? __frcp_rn(s) : 0.f;            // correctly rounded reciprocal
  packed = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int q = static_cast<int>(fminf(fmaxf(rintf(__fmul_rn(v[j], rs)), -8.f), 7.f));
    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * j);
  }
  sb_out = sb;
}

__global__ void __launch_bounds__(256) quant_int4_kernel(const uint16_t* __restrict__ w, long long rows, int cols,
                                                          int rotate, uint8_t* __restrict__ codes,
                                                          uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long u0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kGroupsPerWarp;
  const int ngrp = cols / 128;
  const long long units = rows * ngrp;
  if (u0 >= units) return;
  uint2 raw[kGroupsPerWarp];
#pragma unroll
  for (int k = 0; k < kGroupsPerWarp; ++k) {
    const long long u = u0 + k;
    if (u < units) {
      const long long row = u / ngrp;
      const int g = static_cast<int>(u - row * ngrp);
      raw[k] = __ldg(reinterpret_cast<const uint2*>(w + row * cols + g * 128 + 4 * lane));
    }
  }
#pragma unroll
  for (int k = 0; k < kGroupsPerWarp; ++k) {
    const long long u = u0 + k;
    if (u >= units) break;                                // warp-uniform
    const long long row = u / ngrp;
    const int g = static_cast<int>(u - row * ngrp);
    float v[4] = {bf16_lo(raw[k].x), bf16_hi(raw[k].x), bf16_lo(raw[k].y), bf16_hi(raw[k].y)};
    uint32_t sb, packed;
    quant_int4_group(v, lane, rotate != 0, sb, packed);
    *reinterpret_cast<uint16_t*>(codes + row * (cols / 2) + g * 64 + 2 * lane) = static_cast<uint16_t>(packed);
    if (lane == 0) scales[row * ngrp + g] = static_cast<uint16_t>(sb);
  }
}

// ---------------------------------------------------------------------------------------------
// NVFP4

// Largest |w| of each Linear, as the bits of a non-negative float (which order like the floats), so
// that atomicMax gives the same result in any order.
__global__ void __launch_bounds__(256) quant_amax_kernel(const uint16_t* __restrict__ w, long long per_mat,
                                                          uint32_t* __restrict__ amax) {
  const int mat = blockIdx.y;
  const uint4* src = reinterpret_cast<const uint4*>(w + static_cast<long long>(mat) * per_mat);
  const long long units = per_mat / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  uint32_t m = 0;
  for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < units; i0 += 4 * stride) {
    uint4 q[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) q[r] = i0 + r * stride < units ? __ldg(src + i0 + r * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const uint32_t ws[4] = {q[r].x, q[r].y, q[r].z, q[r].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = max(m, (ws[k] << 16) & 0x7FFFFFFFu);
        m = max(m, ws[k] & 0x7FFF0000u);
      }
    }
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) m = max(m, __shfl_xor_sync(kFull, m, s));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(amax + mat, m);
}

__device__ __forceinline__ float tensor_scale(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? __fdiv_rn(a, 2688.0f) : 1.0f;            // 6 * 448
}

// Non-negative fp32 -> E4M3 (fn) byte, nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rne_pos(float x) {
  if (!(x < 448.0f)) return 0x7Eu;
  if (x < 0.015625f) return static_cast<uint32_t>(rintf(x * 512.0f));   // subnormal steps of 2^-9; 8 = 2^-6
  const uint32_t u = __float_as_uint(x);
  int e = static_cast<int>((u >> 23) & 0xFFu) - 127;                    // x = M 2^e, M in [1, 2)
  float q = rintf(__uint_as_float((u & 0x007FFFFFu) | 0x3F800000u) * 8.0f);   // 8 .. 16
  if (q == 16.0f) {
    ++e;
    q = 8.0f;
  }
  const uint32_t code = (static_cast<uint32_t>(e + 7) << 3) | (static_cast<uint32_t>(q) - 8u);
  return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;              // m 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));               // (1 + m/8) 2^(e-7)
}

// fp32 -> E2M1 nibble: nearest of 0, .5, 1, 1.5, 2, 3, 4, 6, ties to the even code, saturating;
// sign bit 3 from the sign bit of x.
__device__ __forceinline__ uint32_t e2m1_rne(float x) {
  const float a = fabsf(x);
  const uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return c | ((__float_as_uint(x) >> 31) << 3);
}

// One thread per 16-block of a row: its E4M3 scale and 16 codes (8 bytes).
__global__ void __launch_bounds__(256) quant_nvfp4_kernel(const uint16_t* __restrict__ w, long long blocks_per_mat,
                                                           long long total_blocks, const uint32_t* __restrict__ amax,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const long long blk = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= total_blocks) return;
  const int mat = static_cast<int>(blk / blocks_per_mat);
  const float ts = tensor_scale(__ldg(amax + mat));
  const uint4* src = reinterpret_cast<const uint4*>(w + blk * 16);
  const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
  const uint32_t ws[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  float v[16];
  float bm = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = bf16_lo(ws[k]);
    v[2 * k + 1] = bf16_hi(ws[k]);
    bm = fmaxf(bm, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
  }
  const uint32_t sb = e4m3_rne_pos(__fdiv_rn(bm, __fmul_rn(6.0f, ts)));
  const float d = __fmul_rn(e4m3_value(sb), ts);
  const float rd = d > 0.f ? __frcp_rn(d) : 0.f;            // correctly rounded reciprocal
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t c = d > 0.f ? e2m1_rne(__fmul_rn(v[k], rd)) : 0u;
    if (k < 8) lo |= c << (4 * k);
    else hi |= c << (4 * (k - 8));
  }
  *reinterpret_cast<uint2*>(codes + blk * 8) = make_uint2(lo, hi);
  scales[blk] = static_cast<uint8_t>(sb);
}

__global__ void quant_tscale_kernel(float* __restrict__ tscale, int n_mats) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m < n_mats) tscale[m] = tensor_scale(__float_as_uint(tscale[m]));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace flint

using namespace flint;

extern "C" flint_status flint_quantize_int4_g128(const void* w, long long rows, int cols, int rotate, void* codes,
                                                 void* scales, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 128 != 0 || (rotate != 0 && rotate != 1)) return FLINT_ERR_INVALID_ARG;
  if (rows == 0) return FLINT_OK;
  if (!w || !codes || !scales || !aligned(w, 16) || !aligned(codes, 2) || !aligned(scales, 2))
    return FLINT_ERR_INVALID_ARG;
  const long long warps = (rows * (cols / 128) + kGroupsPerWarp - 1) / kGroupsPerWarp;
  const long long grid = (warps + 7) / 8;
  if (grid > 0x7FFFFFFFLL) return FLINT_ERR_INVALID_ARG;
  quant_int4_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(w), rows, cols, rotate, static_cast<uint8_t*>(codes),
      static_cast<uint16_t*>(scales));
  return cudaGetLastError() == cudaSuccess ? FLINT_OK : FLINT_ERR_CUDA;
}

extern "C" flint_status flint_quantize_nvfp4(const void* w, int n_mats, int rows, int cols, void* codes, void* scales,
                                             float* tscale, void* stream) {
  if (n_mats < 0 || n_mats > 65535 || rows < 0 || cols <= 0 || cols % 16 != 0) return FLINT_ERR_INVALID_ARG;
  if (n_mats == 0) return FLINT_OK;
  if (rows == 0) return FLINT_ERR_INVALID_ARG;
  if (!w || !codes || !scales || !tscale || !aligned(w, 16) || !aligned(codes, 8) || !aligned(tscale, 4))
    return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long per_mat = static_cast<long long>(rows) * cols;
  const long long blocks_per_mat = per_mat / 16, total = blocks_per_mat * n_mats;
  if ((total + 255) / 256 > 0x7FFFFFFFLL) return FLINT_ERR_INVALID_ARG;
  uint32_t* amax = reinterpret_cast<uint32_t*>(tscale);        // scratch until quant_tscale_kernel
  if (cudaMemsetAsync(amax, 0, sizeof(uint32_t) * n_mats, s) != cudaSuccess) return FLINT_ERR_CUDA;
  const long long units = per_mat / 8;
  const long long gx = (units + 4095) / 4096;
  quant_amax_kernel<<<dim3(static_cast<unsigned>(gx < 4096 ? gx : 4096), n_mats), 256, 0, s>>>(
      static_cast<const uint16_t*>(w), per_mat, amax);
  quant_nvfp4_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      static_cast<const uint16_t*>(w), blocks_per_mat, total, amax, static_cast<uint8_t*>(codes),
      static_cast<uint8_t*>(scales));
  quant_tscale_kernel<<<(n_mats + 255) / 256, 256, 0, s>>>(tscale, n_mats);
  return cudaGetLastError() == cudaSuccess ? FLINT_OK : FLINT_ERR_CUDA;
}
