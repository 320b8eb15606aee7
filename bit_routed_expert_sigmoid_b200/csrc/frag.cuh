// Warp-level MMA fragment plumbing for the weight-streaming projections.
//
// A thread (lane = 4g + t) of an m16n8k16 MMA owns weight rows g and g+8 of a 16-row tile and token
// column g of the activations. Inside one 128-wide K group, thread t covers 32 consecutive stored
// elements starting at 32t; MMA step i (0..7) takes its 4 stored elements 4i..4i+3. The activation
// operand uses the same stored order, so every product pairs the right weight and activation.
#pragma once

#include "common.cuh"

namespace flint {

// ---- A-fragment sources --------------------------------------------------------------------

// One 128-wide K group of two rows for a thread: raw storage loaded with streaming loads.
template <int FMT>
struct RawA;

template <>
struct RawA<kInt4> {
  uint4 r0, r1;  // 32 codes of row g, row g+8
  __device__ __forceinline__ void load(const uint8_t* row0, const uint8_t* row1, int j, int t) {
    r0 = ld_stream_v4(row0 + j * 64 + 16 * t);
    r1 = ld_stream_v4(row1 + j * 64 + 16 * t);
  }
};

template <>
struct RawA<kNvfp4> {
  uint4 r0, r1;
  __device__ __forceinline__ void load(const uint8_t* row0, const uint8_t* row1, int j, int t) {
    r0 = ld_stream_v4(row0 + j * 64 + 16 * t);
    r1 = ld_stream_v4(row1 + j * 64 + 16 * t);
  }
};

template <>
struct RawA<kBf16> {
  uint4 r0[4], r1[4];  // 32 bf16 of row g, row g+8
  __device__ __forceinline__ void load(const uint8_t* row0, const uint8_t* row1, int j, int t) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      r0[q] = ld_stream_v4(row0 + (j * 128 + 32 * t) * 2 + 16 * q);
      r1[q] = ld_stream_v4(row1 + (j * 128 + 32 * t) * 2 + 16 * q);
    }
  }
};

// 4-bit codes of rows g and g+8 from shared memory (row pointers into a staged tile).
template <int FMT>
__device__ __forceinline__ void load_a_smem(RawA<FMT>& A, const uint8_t* row0, const uint8_t* row1, int j, int t) {
  static_assert(FMT == kInt4 || FMT == kNvfp4, "4-bit formats only");
  A.r0 = *reinterpret_cast<const uint4*>(row0 + j * 64 + 16 * t);
  A.r1 = *reinterpret_cast<const uint4*>(row1 + j * 64 + 16 * t);
}

// bf16 rows g and g+8 from shared memory (row1 == nullptr: row g+8 of the tile is zero).
__device__ __forceinline__ void load_a_bf16_smem(RawA<kBf16>& A, const uint8_t* row0, const uint8_t* row1, int j,
                                                 int t) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    A.r0[q] = *reinterpret_cast<const uint4*>(row0 + (j * 128 + 32 * t) * 2 + 16 * q);
    A.r1[q] = row1 ? *reinterpret_cast<const uint4*>(row1 + (j * 128 + 32 * t) * 2 + 16 * q) : make_uint4(0, 0, 0, 0);
  }
}

// bf16 row g from global memory, row g+8 of the MMA tile left at zero (8-row tiles).
__device__ __forceinline__ void load_a_bf16_one(RawA<kBf16>& A, const uint8_t* row0, int j, int t) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    A.r0[q] = ld_stream_v4(row0 + (j * 128 + 32 * t) * 2 + 16 * q);
    A.r1[q] = make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

// B operand of one group for one thread: 32 stored activations (64 bytes) of token column g.
struct RawB {
  uint4 u[4];
  __device__ __forceinline__ void load(const void* row, int j, int t, bool valid) {
    if (valid) {
      const uint8_t* p = static_cast<const uint8_t*>(row) + (j * 128 + 32 * t) * 2;
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = ld_nc_v4(p + 16 * q);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = make_uint4(0, 0, 0, 0);
    }
  }
  // same, through L2 only (activations written earlier in the same kernel by other CTAs)
  __device__ __forceinline__ void load_cg(const void* row, int j, int t, bool valid) {
    if (valid) {
      const uint8_t* p = static_cast<const uint8_t*>(row) + (j * 128 + 32 * t) * 2;
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = ld_cg_v4(p + 16 * q);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = make_uint4(0, 0, 0, 0);
    }
  }
  // step i uses stored elements 4i..4i+3
  __device__ __forceinline__ uint32_t b0(int i) const { return (i & 1) ? u[i >> 1].z : u[i >> 1].x; }
  __device__ __forceinline__ uint32_t b1(int i) const { return (i & 1) ? u[i >> 1].w : u[i >> 1].y; }
};

// Accumulates one 128-wide group of K into c (fp32) for rows g, g+8 and token columns 2t, 2t+1.
// int4: the group scales sc0/sc1 (rows g, g+8) multiply the group's fp32 partial sums.
// nvfp4: bs0/bs1 point at the rows' E4M3 block scales; codes x block scale are exact in fp16.
// The eight MMA steps accumulate into four independent partial sums (step i into part[i % 4]),
// added in a fixed order at the end: a single accumulator would chain eight dependent MMAs.
template <int FMT, bool TWO_B>
__device__ __forceinline__ void mma_group(float (&c)[4], const RawA<FMT>& A, const RawB& B, const RawB* B2, int j,
                                          int t, float sc0, float sc1, const uint8_t* bs0, const uint8_t* bs1) {
  float part[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int q = 0; q < 4; ++q) part[a][q] = 0.f;
  if constexpr (FMT == kInt4) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t p0[4], p1[4];
      int4x8_to_half2x4(u4_word(A.r0, w), p0);
      int4x8_to_half2x4(u4_word(A.r1, w), p1);
      {
        const uint32_t a[4] = {p0[0], p1[0], p0[1], p1[1]};
        mma_f16_16816(part[(2 * w) & 3], a, B.b0(2 * w), B.b1(2 * w));
      }
      {
        const uint32_t a[4] = {p0[2], p1[2], p0[3], p1[3]};
        mma_f16_16816(part[(2 * w + 1) & 3], a, B.b0(2 * w + 1), B.b1(2 * w + 1));
      }
    }
  } else if constexpr (FMT == kNvfp4) {
    // the thread's 32 codes span two 16-column blocks: steps 0..3 and 4..7
    const int blk = j * 8 + 2 * t;
    uint32_t s0[2], s1[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t h0 = e4m3_to_half_bits(bs0[blk + q]);
      const uint32_t h1 = e4m3_to_half_bits(bs1[blk + q]);
      s0[q] = h0 | (h0 << 16);
      s1[q] = h1 | (h1 << 16);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w0 = u4_word(A.r0, i >> 1), w1 = u4_word(A.r1, i >> 1);
      const int sh = (i & 1) * 16;
      const uint32_t a0 = hmul2_u32(e2m1x2_to_half2(w0 >> sh), s0[i >> 2]);
      const uint32_t a2 = hmul2_u32(e2m1x2_to_half2(w0 >> (sh + 8)), s0[i >> 2]);
      const uint32_t a1 = hmul2_u32(e2m1x2_to_half2(w1 >> sh), s1[i >> 2]);
      const uint32_t a3 = hmul2_u32(e2m1x2_to_half2(w1 >> (sh + 8)), s1[i >> 2]);
      const uint32_t a[4] = {a0, a1, a2, a3};
      mma_f16_16816(part[i & 3], a, B.b0(i), B.b1(i));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a[4] = {u4_word(A.r0[i >> 1], (2 * i) & 3), u4_word(A.r1[i >> 1], (2 * i) & 3),
                             u4_word(A.r0[i >> 1], (2 * i + 1) & 3), u4_word(A.r1[i >> 1], (2 * i + 1) & 3)};
      mma_bf16_16816(part[i & 3], a, B.b0(i), B.b1(i));
      if constexpr (TWO_B) mma_bf16_16816(part[(i + 2) & 3], a, B2->b0(i), B2->b1(i));
    }
  }
  float sum[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) sum[q] = (part[0][q] + part[1][q]) + (part[2][q] + part[3][q]);
  if constexpr (FMT == kInt4) {
    c[0] = fmaf(sc0, sum[0], c[0]);
    c[1] = fmaf(sc0, sum[1], c[1]);
    c[2] = fmaf(sc1, sum[2], c[2]);
    c[3] = fmaf(sc1, sum[3], c[3]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) c[q] += sum[q];
  }
}

// Fixed-order split-K reduction: warps ks = 0..KS-1 of row tile rt add their fragments in order.
template <int KS>
__device__ __forceinline__ bool reduce_splitk(float (&c)[4], float* red, int rt, int ks, int lane) {
  float* mine = red + ((rt * KS + ks) * 32 + lane) * 4;
  if (ks != 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) mine[q] = c[q];
  }
  __syncthreads();
  if (ks != 0) return false;
#pragma unroll
  for (int w = 1; w < KS; ++w) {
    const float* o = red + ((rt * KS + w) * 32 + lane) * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) c[q] += o[q];
  }
  return true;
}


// Same reduction among the first KS*RT warps of a CTA that synchronise on named barrier `bar_id`
// with `nthreads` threads (the consumer warps of a warp-specialised kernel).
template <int KS>
__device__ __forceinline__ bool reduce_splitk_named(float (&c)[4], float* red, int rt, int ks, int lane, int bar_id,
                                                    int nthreads) {
  float* mine = red + ((rt * KS + ks) * 32 + lane) * 4;
  if (ks != 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) mine[q] = c[q];
  }
  named_bar_sync(bar_id, nthreads);
  if (ks != 0) return false;
#pragma unroll
  for (int w = 1; w < KS; ++w) {
    const float* o = red + ((rt * KS + w) * 32 + lane) * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) c[q] += o[q];
  }
  return true;
}

}  // namespace flint
