// Expert projections for small token counts (decode): weight-streaming GEMVs.
//
// Each warp owns a 16-row weight tile and a slice of K; every thread streams 16-byte pieces of
// two rows (row g and row g+8 of the tile, g = lane/4), decodes them in registers to exact fp16
// (int4: code; NVFP4: code x block scale) or uses them as they are (bf16), and feeds them with
// the activations of up to 8 tokens to m16n8k16 tensor-core dot products accumulating in fp32.
// The K order inside an MMA step is a permutation of the stored order; the activation buffers
// are laid out with the same permutation, so every product pairs the right weight and activation.
// Split-K partial sums are reduced through shared memory in a fixed warp order (deterministic).
#include "frag.cuh"
#include "kernels.cuh"

namespace flint {


// ---------------------------------------------------------------------------------------------
// Routed gate|up projection + SwiGLU. Grid (group slot, I/8): the CTA owns 8 gate rows and the 8
// matching up rows of one active expert (a 16-row MMA tile: rows 0..7 gate, 8..15 up) and all of
// K (8 warps x 2 groups). Output h[p][i] in fp32 for the expert's permuted positions p.
template <int FMT>
__global__ void __launch_bounds__(256) gu_routed_kernel(GemvRouted a) {
  __shared__ float red[8 * 32 * 4];
  const int gi = blockIdx.x;
  if (gi >= *a.n_active) return;
  const int e = a.active[gi];
  const int off = a.offsets[e], n = a.offsets[e + 1] - off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int i0 = blockIdx.y * 8;
  const size_t row_bytes = kH / 2;
  const uint8_t* base = a.codes + static_cast<size_t>(e) * (2 * kI) * row_bytes;
  const uint8_t* row0 = base + static_cast<size_t>(i0 + g) * row_bytes;          // gate row
  const uint8_t* row1 = base + static_cast<size_t>(kI + i0 + g) * row_bytes;     // up row
  constexpr int kGroups = kH / kGroup / 8;                                        // 2 per warp
  RawA<FMT> A[kGroups];
  float sc0[kGroups], sc1[kGroups];
  const uint8_t *bs0 = nullptr, *bs1 = nullptr;
#pragma unroll
  for (int q = 0; q < kGroups; ++q) A[q].load(row0, row1, warp * kGroups + q, t);
  if constexpr (FMT == kInt4) {
    const uint16_t* s = static_cast<const uint16_t*>(a.scales) + static_cast<size_t>(e) * (2 * kI) * (kH / kGroup);
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int j = warp * kGroups + q;
      sc0[q] = bf16_bits_to_f32(s[static_cast<size_t>(i0 + g) * (kH / kGroup) + j]);
      sc1[q] = bf16_bits_to_f32(s[static_cast<size_t>(kI + i0 + g) * (kH / kGroup) + j]);
    }
  } else {
    const uint8_t* s = static_cast<const uint8_t*>(a.scales) + static_cast<size_t>(e) * (2 * kI) * (kH / 16);
    bs0 = s + static_cast<size_t>(i0 + g) * (kH / 16);
    bs1 = s + static_cast<size_t>(kI + i0 + g) * (kH / 16);
  }
  float tsg = 1.f, tsu = 1.f;
  if (a.tscale) { tsg = a.tscale[2 * e]; tsu = a.tscale[2 * e + 1]; }

  for (int c0 = 0; c0 < n; c0 += 8) {
    const int nc = min(8, n - c0);
    const bool valid = g < nc;
    const int tok = valid ? a.perm[off + c0 + g] / a.top_k : 0;
    const __half* xrow = a.xq + static_cast<size_t>(tok) * kH;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int j = warp * kGroups + q;
      RawB B;
      B.load(xrow, j, t, valid);
      mma_group<FMT, false>(c, A[q], B, nullptr, j, t, FMT == kInt4 ? sc0[q] : 0.f, FMT == kInt4 ? sc1[q] : 0.f,
                            bs0, bs1);
    }
    if (reduce_splitk<8>(c, red, 0, warp, lane)) {
      // c0/c1: gate row i0+g at tokens 2t, 2t+1; c2/c3: up row i0+g at the same tokens
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int col = 2 * t + q;
        if (col < nc) {
          const float gv = c[q] * tsg, uv = c[2 + q] * tsu;
          a.h_out[static_cast<size_t>(off + c0 + col) * kI + i0 + g] = silu(gv) * uv;
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Routed down projection. Grid (group slot, H/32): the CTA owns 32 output rows (two 16-row tiles)
// of one active expert; warps = 2 tiles x 4 K-groups (K = 512). The CTA first builds the down
// input of each slot in shared memory: h rotated per 128-segment (int4) or h (NVFP4), in fp16.
template <int FMT>
__global__ void __launch_bounds__(256) dn_routed_kernel(GemvRouted a) {
  constexpr int kHs = kI + 8;            // padded fp16 row of the staged down input
  __shared__ float red[8 * 32 * 4];
  __shared__ __align__(16) __half hb[8][kHs];
  const int gi = blockIdx.x;
  if (gi >= *a.n_active) return;
  const int e = a.active[gi];
  const int off = a.offsets[e], n = a.offsets[e + 1] - off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rt = warp >> 2, ks = warp & 3;
  const int n0 = blockIdx.y * 32 + rt * 16;
  const size_t row_bytes = kI / 2;
  const uint8_t* base = a.codes + static_cast<size_t>(e) * kH * row_bytes;
  const uint8_t* row0 = base + static_cast<size_t>(n0 + g) * row_bytes;
  const uint8_t* row1 = base + static_cast<size_t>(n0 + g + 8) * row_bytes;
  RawA<FMT> A;
  A.load(row0, row1, ks, t);                       // issue the weight loads before staging h
  float sc0 = 0.f, sc1 = 0.f;
  const uint8_t *bs0 = nullptr, *bs1 = nullptr;
  if constexpr (FMT == kInt4) {
    const uint16_t* s = static_cast<const uint16_t*>(a.scales) + static_cast<size_t>(e) * kH * (kI / kGroup);
    sc0 = bf16_bits_to_f32(s[static_cast<size_t>(n0 + g) * (kI / kGroup) + ks]);
    sc1 = bf16_bits_to_f32(s[static_cast<size_t>(n0 + g + 8) * (kI / kGroup) + ks]);
  } else {
    const uint8_t* s = static_cast<const uint8_t*>(a.scales) + static_cast<size_t>(e) * kH * (kI / 16);
    bs0 = s + static_cast<size_t>(n0 + g) * (kI / 16);
    bs1 = s + static_cast<size_t>(n0 + g + 8) * (kI / 16);
  }
  const float ts = a.tscale ? a.tscale[e] : 1.f;

  for (int c0 = 0; c0 < n; c0 += 8) {
    const int nc = min(8, n - c0);
    // stage: 8 slots x 4 segments, one warp per (slot, segment)
    for (int w = warp; w < 8 * (kI / kGroup); w += 8) {
      const int slot = w >> 2, seg = w & 3;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (slot < nc) {
        const float4 hv = *reinterpret_cast<const float4*>(a.h_in + static_cast<size_t>(off + c0 + slot) * kI +
                                                           seg * kGroup + 4 * lane);
        v[0] = hv.x; v[1] = hv.y; v[2] = hv.z; v[3] = hv.w;
        if (FMT == kInt4) fwht128_warp(v);
      }
      store_seg_half(&hb[slot][seg * kGroup], v, FMT == kInt4);
    }
    __syncthreads();
    RawB B;
    {
      const uint8_t* p = reinterpret_cast<const uint8_t*>(&hb[g][0]) + (ks * 128 + 32 * t) * 2;
#pragma unroll
      for (int q = 0; q < 4; ++q) B.u[q] = *reinterpret_cast<const uint4*>(p + 16 * q);
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    mma_group<FMT, false>(c, A, B, nullptr, ks, t, sc0, sc1, bs0, bs1);
    if (reduce_splitk<4>(c, red, rt, ks, lane)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 2 * t + (q & 1);
        const int row = n0 + g + 8 * (q >> 1);
        if (col < nc) a.o_out[static_cast<size_t>(off + c0 + col) * kH + row] = c[q] * ts;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Shared expert gate|up + SwiGLU (bf16 weights, bf16 x: exact products, fp32 accumulation).
// Grid Is/8: 8 gate rows + 8 up rows per CTA, all tokens in chunks of 8. hs is stored as a bf16
// pair (hi, lo) with hi + lo = hs to about 16 bits, so the down projection can stay in bf16 MMA.
__global__ void __launch_bounds__(256) gu_shared_kernel(GemvShared a) {
  __shared__ float red[8 * 32 * 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int i0 = blockIdx.x * 8;
  const size_t row_bytes = kH * 2;
  const uint8_t* row0 = a.w_gu + static_cast<size_t>(i0 + g) * row_bytes;
  const uint8_t* row1 = a.w_gu + static_cast<size_t>(kIs + i0 + g) * row_bytes;
  constexpr int kGroups = kH / kGroup / 8;
  RawA<kBf16> A[kGroups];
#pragma unroll
  for (int q = 0; q < kGroups; ++q) A[q].load(row0, row1, warp * kGroups + q, t);
  for (int c0 = 0; c0 < a.T; c0 += 8) {
    const int nc = min(8, a.T - c0);
    const bool valid = g < nc;
    const uint16_t* xrow = a.x + static_cast<size_t>(valid ? c0 + g : 0) * kH;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      RawB B;
      B.load(xrow, warp * kGroups + q, t, valid);
      mma_group<kBf16, false>(c, A[q], B, nullptr, 0, t, 0.f, 0.f, nullptr, nullptr);
    }
    if (reduce_splitk<8>(c, red, 0, warp, lane)) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int col = 2 * t + q;
        if (col < nc) {
          const float hs = silu(c[q]) * c[2 + q];
          const uint16_t hi = f32_to_bf16_bits(hs);
          const uint16_t lo = f32_to_bf16_bits(hs - bf16_bits_to_f32(hi));
          const size_t idx = static_cast<size_t>(c0 + col) * kIs + i0 + g;
          a.hs_hi[idx] = hi;
          a.hs_lo[idx] = lo;
        }
      }
    }
    __syncthreads();
  }
}

// Shared expert down: ys[t][n] = Sd[n] . (hs_hi[t] + hs_lo[t]). Grid H/16, 8 warps = 8 K-groups.
__global__ void __launch_bounds__(256) dn_shared_kernel(GemvShared a) {
  __shared__ float red[8 * 32 * 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * 16;
  const size_t row_bytes = kIs * 2;
  RawA<kBf16> A;
  A.load(a.w_dn + static_cast<size_t>(n0 + g) * row_bytes, a.w_dn + static_cast<size_t>(n0 + g + 8) * row_bytes, warp, t);
  for (int c0 = 0; c0 < a.T; c0 += 8) {
    const int nc = min(8, a.T - c0);
    const bool valid = g < nc;
    const size_t r = static_cast<size_t>(valid ? c0 + g : 0) * kIs;
    RawB Bh, Bl;
    Bh.load(a.hs_hi + r, warp, t, valid);
    Bl.load(a.hs_lo + r, warp, t, valid);
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    mma_group<kBf16, true>(c, A, Bh, &Bl, 0, t, 0.f, 0.f, nullptr, nullptr);
    if (reduce_splitk<8>(c, red, 0, warp, lane)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 2 * t + (q & 1);
        const int row = n0 + g + 8 * (q >> 1);
        if (col < nc) a.ys[static_cast<size_t>(c0 + col) * kH + row] = c[q];
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Combine: y[t][n] = bf16( routed_scale * sum_k w[t][k] * o[inv[t][k]][n] + ys[t][n] ), the slots
// summed in slot order (ascending expert id), one rounding at the end.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o, const float* __restrict__ ys,
                                                      const float* __restrict__ w, const int* __restrict__ inv,
                                                      int K, float routed_scale, uint16_t* __restrict__ y) {
  const int t = blockIdx.y;
  const int n = (blockIdx.x * 256 + threadIdx.x) * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < K; ++k) {
    const float wk = w[t * K + k];
    const float4 ov = *reinterpret_cast<const float4*>(o + static_cast<size_t>(inv[t * K + k]) * kH + n);
    acc[0] = fmaf(wk, ov.x, acc[0]);
    acc[1] = fmaf(wk, ov.y, acc[1]);
    acc[2] = fmaf(wk, ov.z, acc[2]);
    acc[3] = fmaf(wk, ov.w, acc[3]);
  }
  const float4 sv = *reinterpret_cast<const float4*>(ys + static_cast<size_t>(t) * kH + n);
  uint2 out;
  out.x = pack_bf162(fmaf(routed_scale, acc[0], sv.x), fmaf(routed_scale, acc[1], sv.y));
  out.y = pack_bf162(fmaf(routed_scale, acc[2], sv.z), fmaf(routed_scale, acc[3], sv.w));
  *reinterpret_cast<uint2*>(y + static_cast<size_t>(t) * kH + n) = out;
}

// ---------------------------------------------------------------------------------------------
// launchers

cudaError_t launch_gu_routed(const GemvRouted& a, int fmt, int groups, cudaStream_t s) {
  dim3 grid(groups, kI / 8);
  if (fmt == kInt4) gu_routed_kernel<kInt4><<<grid, 256, 0, s>>>(a);
  else gu_routed_kernel<kNvfp4><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dn_routed(const GemvRouted& a, int fmt, int groups, cudaStream_t s) {
  dim3 grid(groups, kH / 32);
  if (fmt == kInt4) dn_routed_kernel<kInt4><<<grid, 256, 0, s>>>(a);
  else dn_routed_kernel<kNvfp4><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gu_shared(const GemvShared& a, cudaStream_t s) {
  gu_shared_kernel<<<kIs / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dn_shared(const GemvShared& a, cudaStream_t s) {
  dn_shared_kernel<<<kH / 16, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* o, const float* ys, const float* w, const int* inv, int T, int K,
                           float routed_scale, uint16_t* y, cudaStream_t s) {
  dim3 grid(kH / 1024, T);
  combine_kernel<<<grid, 256, 0, s>>>(o, ys, w, inv, K, routed_scale, y);
  return cudaGetLastError();
}

}  // namespace flint
