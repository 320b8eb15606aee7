// NVFP4 weights x NVFP4 activations (W4A4) for large token counts (prefill).
//
// kekzle/Flint-NVFP4, evaluation table and serving notes: in prefill the activations entering each
// routed projection are quantised to NVFP4 as well, and the projections run on the FP4 tensor cores.
// Here that is:
//   act_quant_*_kernel  a row (a token's x, written to its top-k permuted rows; or a permuted row of
//                       the SwiGLU output h) -> E2M1 codes, one E4M3 scale per 16 values and one fp32
//                       scale per row (amax / (6 x 448)); every decision in IEEE fp32, in the order
//                       ts, block scale, quotient, code
//   w4a4_kernel         routed grouped GEMM on tcgen05.mma kind::mxf4nvf4 (block16: E2M1 operands
//                       from shared memory, E4M3 scales from tensor memory, fp32 accumulators in
//                       tensor memory); epilogue x (weight scale x activation scale); gate|up ->
//                       h = silu(g) u in fp32, down -> o in fp16 (combined per token by the prefill
//                       combine kernel)
//
// Scale layout of one MMA (K = 64, four 16-blocks): row m = m0 + 32 m1 of an operand (m0 < 32,
// m1 < 4) has its four E4M3 scales as bytes 0..3 of tensor-memory column m1 in lane m0, copied to
// all four lane quarters by tcgen05.cp .32x128b.warpx4 from a 512-byte "atom" whose 16-byte row m0
// holds [m1][block]. The scales are stored in that layout ahead of the GEMM, so a stage (four
// K-steps) of a 128-row weight block or of a 64-row activation chunk is one contiguous 2 KB copy:
//   weights      [row block of 128][K/64][atom], packed once when the handle is made
//                (pack_sf_atoms_kernel) from the [row][K/16] scales
//   activations  [chunk][K/64][atom], written by the quantisers; a chunk is 64 consecutive permuted
//                rows of one expert (the GEMM's N), numbered over all experts in ascending order (the
//                permutation kernel writes each expert's first chunk), and only m1 = 0, 1 of its atoms
//                are meaningful
//
// The routed GEMM walks the tile table of the W4A16 routed kernel: a tile is (expert, a chunk of up
// to 64 of its permuted rows, a pair of 128-row weight blocks). One persistent CTA per SM; warps:
//   warp 0      TMA: the pair of weight-code blocks (128 rows x 128 bytes = 256 K, 128-byte swizzle)
//               and a bulk copy of each block's scale atoms, per stage
//   warp 3      TMA: the chunk's activation codes (16-row boxes) and a bulk copy of its scale atoms;
//               after griddepcontrol.wait, as they are the previous kernel's output
//   warps 1, 2  MMA issue, one warp per weight block: tcgen05.cp of the block's and the chunk's
//               atoms into the warp's own tensor-memory columns, then the block's four MMAs; warp 1
//               also owns the tensor-memory allocation
//   warps 4..11 epilogue, two per 32-lane quarter of tensor memory (warp w reads lanes 32 (w % 4)..),
//               warps 4..7 the 16-column groups 0 and 2 of a tile, warps 8..11 groups 1 and 3; the
//               accumulators are released as soon as they are in registers
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace flint {

namespace {

constexpr int kAtom = 512;                         // bytes of one scale atom (one MMA K-step)

// ---------------------------------------------------------------------------------------------
// activation quantisers

__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float q) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) { return __half2float(__ushort_as_half(e4m3_to_half_bits(byte))); }

// (first, second) -> one byte of two E2M1 codes, the first in the low nibble (nearest, ties to
// even, saturating at 6)
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float first, float second) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(second), "f"(first));
  return r;
}

// Eight values of a row (half of a 16-block; the other half is in lane ^ 1) -> their four code
// bytes as one word; `sb` gets the block's E4M3 scale.
__device__ __forceinline__ uint32_t quant8(const float (&v)[8], float ts, uint32_t& sb) {
  float bm = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) bm = fmaxf(bm, fabsf(v[i]));
  bm = fmaxf(bm, __shfl_xor_sync(kAll, bm, 1));
  sb = f32_to_e4m3_satfinite(__fdiv_rn(bm, __fmul_rn(6.f, ts)));
  const float d = __fmul_rn(e4m3_to_f32(sb), ts);
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = v[2 * i], b = v[2 * i + 1];
    const uint32_t byte = d > 0.f ? f32x2_to_e2m1x2(__fdiv_rn(a, d), __fdiv_rn(b, d))
                                  : (signbit(a) ? 0x8u : 0u) | (signbit(b) ? 0x80u : 0u);
    w |= byte << (8 * i);
  }
  return w;
}

// The four block scales of a K-step (16-blocks held by lanes g, g + 2, g + 4, g + 6 of the 8-lane
// group g) as one word, the first block in the low byte.
__device__ __forceinline__ uint32_t kstep_scales(uint32_t sb, int lane) {
  const int g = lane & ~7;
  return __shfl_sync(kAll, sb, g) | (__shfl_sync(kAll, sb, g + 2) << 8) | (__shfl_sync(kAll, sb, g + 4) << 16) |
         (__shfl_sync(kAll, sb, g + 6) << 24);
}

// One quantised row (thread i holds values 8i..8i+7 of K) to its destination: codes, raw scales,
// tensor scale, and the scale atoms of its chunk position pos = chunk * 64 + row in chunk.
template <int K>
__device__ __forceinline__ void store_row(int i, int lane, size_t dst, int pos, uint32_t w, uint32_t sb, uint32_t step_sc,
                                          float ts, uint8_t* codes, uint8_t* scales, uint8_t* atoms, float* ts_out) {
  reinterpret_cast<uint32_t*>(codes + dst * (K / 2))[i] = w;
  if ((i & 1) == 0) scales[dst * (K / 16) + (i >> 1)] = static_cast<uint8_t>(sb);
  if ((lane & 7) == 0) {
    const int c = pos >> 6, n = pos & 63, j = i >> 3;
    *reinterpret_cast<uint32_t*>(atoms + (static_cast<size_t>(c) * (K / 64) + j) * kAtom + (n & 31) * 16 + (n >> 5) * 4) =
        step_sc;
  }
  if (i == 0) ts_out[dst] = ts;
}

// Row amax over the K / 8 threads of a row (whole warps), then the row's tensor scale.
template <int K>
__device__ __forceinline__ float row_tscale(const float (&v)[8], float* wmax, int lr, int warp, int lane) {
  constexpr int kWpr = K / 8 / 32;
  float am = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) am = fmaxf(am, __shfl_xor_sync(kAll, am, d));
  if (lane == 0) wmax[warp] = am;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kWpr; ++k) am = fmaxf(am, wmax[lr * kWpr + k]);
  return am > 0.f ? __fdiv_rn(am, 2688.f) : 1.f;
}

// x: one token per CTA (256 threads x 8 values). Warp 0 first places each of the token's top-k
// permuted rows in its expert's 64-row chunks (chunk_base from the permutation kernel): its chunk
// position, also stored in rowc for the h quantiser.
__global__ void __launch_bounds__(256) act_quant_x_kernel(const uint16_t* __restrict__ x, int top_k, int E,
                                                          const int* __restrict__ ids, const int* __restrict__ inv,
                                                          const int* __restrict__ offsets,
                                                          const int* __restrict__ chunk_base, uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ scales, uint8_t* __restrict__ atoms,
                                                          float* __restrict__ ts_out, int* __restrict__ rowc) {
  static_assert(kH / 8 == 256, "one token per 256 threads");
  __shared__ float wmax[8];
  __shared__ int dst_row[kMaxTopK], dst_pos[kMaxTopK];
  const int t = blockIdx.x, i = threadIdx.x, warp = i >> 5, lane = i & 31;
  pdl_wait();                                      // ids, inv, offsets and chunk_base: the permutation's output
  pdl_trigger();
  if (warp == 0 && lane < top_k) {
    const int e = min(max(__ldg(ids + t * top_k + lane), 0), E - 1);
    const int p = __ldg(inv + t * top_k + lane);
    const int local = p - __ldg(offsets + e);
    const int pos = (__ldg(chunk_base + e) + (local >> 6)) * 64 + (local & 63);
    dst_row[lane] = p;
    dst_pos[lane] = pos;
    rowc[p] = pos;
  }
  float v[8];
  const uint4 wx = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * kH) + i);
  const uint32_t u[4] = {wx.x, wx.y, wx.z, wx.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = bf16lo_to_f32(u[j]);
    v[2 * j + 1] = bf16hi_to_f32(u[j]);
  }
  const float ts = row_tscale<kH>(v, wmax, 0, warp, lane);     // its __syncthreads also publishes dst_*
  uint32_t sb;
  const uint32_t w = quant8(v, ts, sb);
  const uint32_t step_sc = kstep_scales(sb, lane);
  for (int k = 0; k < top_k; ++k)
    store_row<kH>(i, lane, static_cast<size_t>(dst_row[k]), dst_pos[k], w, sb, step_sc, ts, codes, scales, atoms, ts_out);
}

// h: permuted rows of I values, 64 threads each, 4 per CTA; the chunk position of row p is rowc[p].
__global__ void __launch_bounds__(256) act_quant_h_kernel(const float* __restrict__ h, int P, const int* __restrict__ rowc,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                          uint8_t* __restrict__ atoms, float* __restrict__ ts_out) {
  constexpr int kTpr = kI / 8, kRows = 256 / kTpr;
  __shared__ float wmax[8];
  const int lr = threadIdx.x / kTpr, i = threadIdx.x % kTpr;
  const int row = blockIdx.x * kRows + lr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();                                      // h is the previous kernel's output
  pdl_trigger();
  float v[8];
  int pos = 0;
  if (row < P) {
    const float4* src = reinterpret_cast<const float4*>(h + static_cast<size_t>(row) * kI) + 2 * i;
    const float4 a = src[0], b = src[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    pos = __ldg(rowc + row);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
  }
  const float ts = row_tscale<kI>(v, wmax, lr, warp, lane);
  uint32_t sb;
  const uint32_t w = quant8(v, ts, sb);
  const uint32_t step_sc = kstep_scales(sb, lane);
  if (row < P) store_row<kI>(i, lane, static_cast<size_t>(row), pos, w, sb, step_sc, ts, codes, scales, atoms, ts_out);
}

// Weight scales [rows][K/16] -> atoms [rows / 128][K/64][512 bytes]: one thread per (row block,
// K-step, m0) writes the 16 bytes of rows m0, m0 + 32, m0 + 64, m0 + 96.
__global__ void pack_sf_atoms_kernel(const uint8_t* __restrict__ sc, int rows, int K, uint8_t* __restrict__ out) {
  const int steps = K / 64;
  const size_t n = static_cast<size_t>(rows / 128) * steps * 32;
  for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m0 = static_cast<int>(idx & 31);
    const size_t q = idx >> 5;
    const int j = static_cast<int>(q % steps);
    const size_t rb = q / steps;
    uint32_t wv[4];
#pragma unroll
    for (int m1 = 0; m1 < 4; ++m1)
      wv[m1] = *reinterpret_cast<const uint32_t*>(sc + (rb * 128 + m0 + 32 * m1) * (K / 16) + 4 * j);
    *reinterpret_cast<uint4*>(out + (rb * steps + j) * kAtom + m0 * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

// ---------------------------------------------------------------------------------------------
// routed grouped GEMM, kind::mxf4nvf4

constexpr int kW4D = 4;                            // ring depth (stages of 256 K)
constexpr int kW4ABox = 128 * 128;                 // weight codes: 128 rows x 128 bytes
constexpr int kW4BRows = kPfN;                     // activation rows per tile (MMA N, up to)
constexpr int kW4StepAtoms = 4 * kAtom;            // a stage's atoms of one operand block (2 KB)
constexpr int kW4OffA = 0;
constexpr int kW4OffB = kW4OffA + 2 * kW4ABox;
constexpr int kW4OffSfA = kW4OffB + kW4BRows * 128;  // atoms of weight blocks 0 and 1
constexpr int kW4OffSfB = kW4OffSfA + 2 * kW4StepAtoms;
constexpr int kW4Stage = kW4OffSfB + kW4StepAtoms;
static_assert(kW4Stage % 1024 == 0 && kW4OffB % 1024 == 0, "128-byte swizzled operands on 1024-byte boundaries");
constexpr int kW4OffTab = kW4D * kW4Stage;
// down epilogue: per epilogue warp a 16-token x 32-output fp16 slab, to turn its column-per-lane
// results into 16-byte row stores
constexpr int kW4OffSlab = (kW4OffTab + static_cast<int>(sizeof(TileTab)) + 15) / 16 * 16;
constexpr int kW4OffBar = kW4OffSlab + 8 * 16 * 32 * 2;

struct W4Bars {
  uint64_t full_a[kW4D], full_b[kW4D], empty[kW4D];
  uint64_t acc_full[2], acc_empty[2], done[2];
  uint32_t tmem;
  int abort;
};
constexpr int kW4Smem = kW4OffBar + static_cast<int>(sizeof(W4Bars)) + 1024;
static_assert(kW4Smem <= 227 * 1024, "shared memory per CTA");

// tensor memory: accumulators [slot 2][block 2] x 64 columns, then per ring slot and weight block
// (the MMA warp that issues it) 16 columns of the block's scales (4 K-steps x 4) and 16 of the
// chunk's
constexpr int kW4Threads = 384;
constexpr uint32_t kW4ColSf = 256;
constexpr uint32_t kW4SfSlot = 64;
static_assert(kW4ColSf + kW4D * kW4SfSlot <= 512, "tensor-memory columns");

template <int PHASE>
struct W4Geom;
template <>
struct W4Geom<kPhaseGateUp> {
  static constexpr int K = kH, S = kH / 256, RP = kI / 128;
  __device__ static int row(int w, int rp, int b) { return w * 2 * kI + b * kI + rp * 128; }
};
template <>
struct W4Geom<kPhaseDown> {
  static constexpr int K = kI, S = kI / 256, RP = kH / 256;
  __device__ static int row(int w, int rp, int b) { return w * kH + rp * 256 + b * 128; }
};

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (K-major), E4M3 scales, M = 128, fp32 D.
__device__ __forceinline__ uint32_t idesc_mxf4nvf4(int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// Shared-memory descriptor of a scale atom for tcgen05.cp: no swizzle, 8-row core matrices of 16
// bytes per row, 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_atom(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 16) |
         (static_cast<uint64_t>(128 >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}

// Warp-wide copy and MMA: one elected lane (the same one for both, so the copies precede the MMAs
// that read them in the tensor pipe's issue order).
__device__ __forceinline__ void tc_cp_atom_w(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}

__device__ __forceinline__ void tc_mma_fp4_w(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                             uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %6, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}

template <int PHASE>
__global__ void __launch_bounds__(kW4Threads, 1) w4a4_kernel(const __grid_constant__ PrefillParams p) {
  using G = W4Geom<PHASE>;
  constexpr int kSteps = G::K / 64;              // atoms per row block / chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  TileTab& tt = *reinterpret_cast<TileTab*>(sm + kW4OffTab);
  W4Bars& bb = *reinterpret_cast<W4Bars*>(sm + kW4OffBar);
  volatile int* abort = &bb.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kW4D; ++i) {
      mbar_init(&bb.full_a[i], 1);
      mbar_init(&bb.full_b[i], 1);
      mbar_init(&bb.empty[i], 2);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bb.acc_full[a], 2);
      mbar_init(&bb.acc_empty[a], 8);
    }
    mbar_init(&bb.done[0], 1);
    mbar_init(&bb.done[1], 1);
    bb.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) build_tiles<true>(tt, p, G::RP);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&bb.tmem)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bb.tmem;
  const int total = tt.total;
  pdl_trigger();

  if (warp == 0) {
    // ---- weight codes and scale atoms (read once: evicted first from L2)
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at<true>(tt, t);
        const int r0 = G::row(tl.w, tl.rp, 0), r1 = G::row(tl.w, tl.rp, 1);
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kW4D;
          if (it >= kW4D && !pf_wait(&bb.empty[slot], ((it / kW4D) - 1) & 1, abort, p.err)) break;
          uint8_t* st = sm + slot * kW4Stage;
          mbar_arrive_expect_tx(&bb.full_a[slot], 2 * kW4ABox + 2 * kW4StepAtoms);
          tma_2d_hint(st + kW4OffA, &p.tm_codes, s * 128, r0, &bb.full_a[slot], pol);
          tma_2d_hint(st + kW4OffA + kW4ABox, &p.tm_codes, s * 128, r1, &bb.full_a[slot], pol);
          bulk_g2s_hint(st + kW4OffSfA, p.w_atoms + (static_cast<size_t>(r0 / 128) * kSteps + 4 * s) * kAtom,
                        kW4StepAtoms, &bb.full_a[slot], pol);
          bulk_g2s_hint(st + kW4OffSfA + kW4StepAtoms,
                        p.w_atoms + (static_cast<size_t>(r1 / 128) * kSteps + 4 * s) * kAtom, kW4StepAtoms,
                        &bb.full_a[slot], pol);
        }
      }
      for (int j = max(it - kW4D, 0); j < it; ++j) pf_wait(&bb.full_a[j % kW4D], (j / kW4D) & 1, abort, p.err);
    }
  } else if (warp == 3) {
    // ---- activation codes (the chunk's rows rounded up to 16) and the chunk's scale atoms
    if (lane == 0) {
      pdl_wait();
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at<true>(tt, t);
        const int nbox = (tl.n + 15) >> 4;
        bool ok = true;
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kW4D;
          if (it >= kW4D && !pf_wait(&bb.empty[slot], ((it / kW4D) - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = sm + slot * kW4Stage;
          mbar_arrive_expect_tx(&bb.full_b[slot], nbox * 16 * 128 + kW4StepAtoms);
          for (int q = 0; q < nbox; ++q)
            tma_2d(st + kW4OffB + q * 2048, &p.tm_act, s * 128, tl.row0 + 16 * q, &bb.full_b[slot]);
          bulk_g2s(st + kW4OffSfB, p.act_atoms + (static_cast<size_t>(tl.c) * kSteps + 4 * s) * kAtom, kW4StepAtoms,
                   &bb.full_b[slot]);
        }
        if (!ok) break;
      }
      for (int j = max(it - kW4D, 0); j < it; ++j) pf_wait(&bb.full_b[j % kW4D], (j / kW4D) & 1, abort, p.err);
    }
  } else if (warp == 1 || warp == 2) {
    // ---- scale copies and MMA issue for one weight block (uniform control flow; an elected lane issues)
    const int b = warp - 1;
    int it = 0, ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
      const PfTile tl = tile_at<true>(tt, t);
      const uint32_t idesc = idesc_mxf4nvf4((tl.n + 15) & ~15);
      const int as = ti & 1;
      if (ti >= 2 && !pf_wait_all(&bb.acc_empty[as], ((ti >> 1) - 1) & 1, abort, p.err)) break;
      tc_fence_after();
      const uint32_t d = tmem + as * 128 + b * 64;
      for (int s = 0; s < G::S; ++s, ++it) {
        const int slot = it % kW4D;
        if (!pf_wait_all(&bb.full_a[slot], (it / kW4D) & 1, abort, p.err) ||
            !pf_wait_all(&bb.full_b[slot], (it / kW4D) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(sm + slot * kW4Stage);
        const uint32_t sfa = tmem + kW4ColSf + slot * kW4SfSlot + b * 32, sfb = sfa + 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tc_cp_atom_w(sfa + j * 4, sdesc_atom(st + kW4OffSfA + b * kW4StepAtoms + j * kAtom));
          tc_cp_atom_w(sfb + j * 4, sdesc_atom(st + kW4OffSfB + j * kAtom));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc_mma_fp4_w(d, sdesc_sw128(st + kW4OffA + b * kW4ABox + j * 32), sdesc_sw128(st + kW4OffB + j * 32),
                       idesc, sfa + j * 4, sfb + j * 4, (s | j) ? 1u : 0u);
        tc_commit_w(&bb.empty[slot]);
      }
      if (ok) tc_commit_w(&bb.acc_full[as]);
    }
    tc_commit_w(&bb.done[b]);                      // every MMA and copy of this warp has completed
    pf_wait_all(&bb.done[b], 0, abort, p.err);
  } else if (warp >= 4 && warp < 12) {
    // ---- epilogue: lane quarter q holds weight rows 32q.. of both blocks; set k the 16-column
    // groups k and k + 2
    const int q = warp & 3, r = 32 * q + lane, k = (warp - 4) >> 2;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    __half* slab = reinterpret_cast<__half*>(sm + kW4OffSlab) + (warp - 4) * 16 * 32;
    pdl_wait();                                    // the activation tensor scales are the previous kernel's output
    // A tile's scales (the weight tensor scales and one activation tensor scale per column, column c
    // in lane c % 32 of ts_lo / ts_hi) are loaded one tile ahead, so their latency is hidden.
    struct Scales {
      float tw0, tw1, ts_lo, ts_hi;
    };
    auto load_scales = [&](const PfTile& tl) {
      Scales sc;
      if constexpr (PHASE == kPhaseGateUp) {
        sc.tw0 = __ldg(p.tscale + 2 * tl.w);
        sc.tw1 = __ldg(p.tscale + 2 * tl.w + 1);
      } else {
        sc.tw0 = sc.tw1 = __ldg(p.tscale + tl.w);
      }
      sc.ts_lo = lane < tl.n ? __ldg(p.act_ts + tl.row0 + lane) : 0.f;
      sc.ts_hi = lane + 32 < tl.n ? __ldg(p.act_ts + tl.row0 + 32 + lane) : 0.f;
      return sc;
    };
    int ti = 0;
    PfTile tl{};
    Scales sc{};
    if (static_cast<int>(blockIdx.x) < total) {
      tl = tile_at<true>(tt, blockIdx.x);
      sc = load_scales(tl);
    }
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++ti) {
      const int as = ti & 1;
      PfTile tn{};
      Scales sn{};
      if (t + static_cast<int>(gridDim.x) < total) {
        tn = tile_at<true>(tt, t + gridDim.x);
        sn = load_scales(tn);
      }
      if (!pf_wait_all(&bb.acc_full[as], (ti >> 1) & 1, abort, p.err)) break;
      tc_fence_after();
      // this warp's column groups (k and k + 2) of both blocks into registers, then the
      // accumulators are released before the math and the stores
      const uint32_t dbase = lane_base + as * 128;
      const int ng = tl.n > 16 * (k + 2) ? 2 : tl.n > 16 * k ? 1 : 0;
      uint32_t dv[2][2][16];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        if (g < ng) {
          tc_ld16(dbase + 16 * (k + 2 * g), dv[g][0]);
          tc_ld16(dbase + 64 + 16 * (k + 2 * g), dv[g][1]);
        }
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bb.acc_empty[as]);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        if (g >= ng) break;
        const int j0 = 16 * (k + 2 * g);
        if constexpr (PHASE == kPhaseGateUp) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float ta = __shfl_sync(kAll, j0 < 32 ? sc.ts_lo : sc.ts_hi, (j0 + c) & 31);
            if (j0 + c < tl.n) {
              const size_t row = static_cast<size_t>(tl.row0 + j0 + c);
              const float v0 = __uint_as_float(dv[g][0][c]) * (sc.tw0 * ta);
              const float v1 = __uint_as_float(dv[g][1][c]) * (sc.tw1 * ta);
              p.h32[row * kI + tl.rp * 128 + r] = silu_fast(v0) * v1;
            }
          }
        } else {
          // o rows through the slab: lane = output (32q + lane of the block), 16 tokens, then each
          // lane stores 16-byte pieces (8 outputs) of two token rows
#pragma unroll
          for (int b = 0; b < 2; ++b) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float ta = __shfl_sync(kAll, j0 < 32 ? sc.ts_lo : sc.ts_hi, (j0 + c) & 31);
              slab[c * 32 + lane] = __float2half_rn(__uint_as_float(dv[g][b][c]) * (sc.tw0 * ta));
            }
            __syncwarp();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int piece = lane + 32 * h, c = piece >> 2, f = (piece & 3) * 8;
              if (j0 + c < tl.n) {
                const uint4 v = *reinterpret_cast<const uint4*>(slab + c * 32 + f);
                *reinterpret_cast<uint4*>(p.o + static_cast<size_t>(tl.row0 + j0 + c) * kH + tl.rp * 256 + b * 128 +
                                          32 * q + f) = v;
              }
            }
            __syncwarp();
          }
        }
      }
      tl = tn;
      sc = sn;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

}  // namespace

size_t w4a4_chunk_capacity(size_t P, int E) { return (P + 63) / 64 + static_cast<size_t>(E); }

cudaError_t launch_pack_sf_atoms(const uint8_t* scales, int rows, int K, uint8_t* atoms, cudaStream_t s) {
  if (rows % 128 != 0 || K % 64 != 0) return cudaErrorInvalidValue;
  const size_t n = static_cast<size_t>(rows / 128) * (K / 64) * 32;
  if (n == 0) return cudaSuccess;
  const int grid = static_cast<int>(std::min<size_t>((n + 255) / 256, 65535));
  pack_sf_atoms_kernel<<<grid, 256, 0, s>>>(scales, rows, K, atoms);
  return cudaGetLastError();
}

cudaError_t launch_act_quant_x(const uint16_t* x, int T, int K, int E, const int* ids, const int* inv,
                               const int* offsets, const int* chunk_base, uint8_t* codes, uint8_t* scales,
                               uint8_t* atoms, float* ts, int* rowc, cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl_kernel(act_quant_x_kernel, T, 256, 0, pdl, s, x, K, E, ids, inv, offsets, chunk_base, codes, scales,
                           atoms, ts, rowc);
}

cudaError_t launch_act_quant_h(const float* h, int P, const int* rowc, uint8_t* codes, uint8_t* scales, uint8_t* atoms,
                               float* ts, bool pdl, cudaStream_t s) {
  if (P <= 0) return cudaSuccess;
  constexpr int kRows = 256 / (kI / 8);
  return launch_pdl_kernel(act_quant_h_kernel, (P + kRows - 1) / kRows, 256, 0, pdl, s, h, P, rowc, codes, scales, atoms,
                           ts);
}

cudaError_t launch_w4a4_routed(const PrefillParams& p, int phase, int n_sm, bool pdl, cudaStream_t s) {
  static bool smem_set = false;
  if (!smem_set) {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(w4a4_kernel<kPhaseGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize, kW4Smem)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(w4a4_kernel<kPhaseDown>, cudaFuncAttributeMaxDynamicSharedMemorySize, kW4Smem)) !=
        cudaSuccess)
      return e;
    smem_set = true;
  }
  return phase == kPhaseGateUp ? launch_pdl_kernel(w4a4_kernel<kPhaseGateUp>, n_sm, kW4Threads, kW4Smem, pdl, s, p)
                               : launch_pdl_kernel(w4a4_kernel<kPhaseDown>, n_sm, kW4Threads, kW4Smem, pdl, s, p);
}

}  // namespace flint
