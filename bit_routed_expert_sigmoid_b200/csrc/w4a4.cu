// NVFP4 weights x NVFP4 activations (W4A4) for large token counts (prefill).
//
// kekzle/Flint-NVFP4, evaluation table and serving notes: in prefill the activations entering each
// routed projection are quantised to NVFP4 as well, and the projections run on the FP4 tensor cores.
// Here that is:
//   act_quant_kernel   a row (a token's x, scattered to its top-k permuted rows; or a permuted row of
//                      the SwiGLU output h) -> E2M1 codes, one E4M3 scale per 16 values and one fp32
//                      scale per row (amax / (6 x 448)); every decision in IEEE fp32, in the order
//                      ts, block scale, quotient, code
//   w4a4_kernel        routed grouped GEMM on tcgen05.mma kind::mxf4nvf4 (block16: E2M1 operands from
//                      shared memory, E4M3 scales from tensor memory, fp32 accumulators in tensor
//                      memory); epilogue x (weight scale x activation scale); gate|up -> h = silu(g) u
//                      in fp32, down -> o in fp16 (combined per token by the prefill combine kernel)
//
// The routed GEMM uses the tile table of the W4A16 routed kernel: a tile is (expert, a chunk of up
// to 64 of its permuted rows, a pair of 128-row weight blocks). One persistent CTA per SM; warps:
//   warp 0      TMA: the pair of weight-code blocks (128 rows x 128 bytes = 256 K, 128-byte swizzle)
//               and their raw block scales (128 rows x 16 bytes) per stage
//   warp 3      TMA: the chunk's activation codes (16-row boxes, 128-byte swizzle) and raw scales;
//               after griddepcontrol.wait, as they are the previous kernel's output
//   warps 2, 13 scale layout: rewrite the raw scales of a stage into the MMA's scale layout (below);
//               warp 2 those of weight block 0 and of the activations, warp 13 those of block 1
//   warps 1, 12 MMA issue, one warp per weight block: tcgen05.cp of the block's and the activations'
//               scales into its own tensor-memory columns, then the block's MMAs; warp 1 also owns
//               the tensor-memory allocation
//   warps 4..11 epilogue, two per 32-lane quarter of tensor memory (warp w reads lanes 32 (w % 4)..),
//               warps 4..7 the even 16-column groups of a tile, warps 8..11 the odd ones (a down
//               tile has only two stages to hide its epilogue behind)
//
// Scale layout of one MMA (K = 64, four 16-blocks): a row m = m0 + 32 m1 of the operand (m0 < 32,
// m1 < 4) has its four E4M3 scales as bytes 0..3 of tensor-memory column m1 in lane m0 (copied to
// all four lane quarters by tcgen05.cp .32x128b.warpx4 from a 512-byte shared-memory atom whose row
// m0 holds 16 bytes: m1-major, block-minor). The raw scales of a weight or activation row are
// contiguous along K ([row][K/16] bytes), so the atom for K-step j takes the j-th 32-bit word of
// rows m0, m0+32, m0+64 and m0+96.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace flint {

namespace {

// ---------------------------------------------------------------------------------------------
// activation quantiser

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

// Rows of K values, 8 values per thread (K / 8 threads per row), 256 threads per CTA.
// SRC_BF16: rows are bf16 tokens, each written to its top_k permuted rows inv[t][k]; else rows are
// fp32 permuted rows written in place.
template <int K, bool SRC_BF16>
__global__ void __launch_bounds__(256) act_quant_kernel(const void* __restrict__ src, int rows, int top_k,
                                                        const int* __restrict__ inv, uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales, float* __restrict__ ts_out) {
  constexpr int kTpr = K / 8;                    // threads per row
  constexpr int kRows = 256 / kTpr;              // rows per CTA
  constexpr int kWpr = (kTpr + 31) / 32;         // warps per row
  static_assert(kTpr % 32 == 0 && kRows >= 1, "whole warps per row");
  __shared__ float wmax[8];
  const int lr = threadIdx.x / kTpr, i = threadIdx.x % kTpr;
  const int row = blockIdx.x * kRows + lr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (!SRC_BF16) pdl_wait();           // h is the previous kernel's output
  pdl_trigger();
  float v[8];
  if (row < rows) {
    if constexpr (SRC_BF16) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + static_cast<size_t>(row) * K) + i);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = bf16lo_to_f32(u[j]);
        v[2 * j + 1] = bf16hi_to_f32(u[j]);
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + static_cast<size_t>(row) * K) + 2 * i;
      const float4 a = p[0], b = p[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
  }
  float am = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) am = fmaxf(am, __shfl_xor_sync(kAll, am, d));
  if (lane == 0) wmax[warp] = am;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kWpr; ++k) am = fmaxf(am, wmax[lr * kWpr + k]);
  const float ts = am > 0.f ? __fdiv_rn(am, 2688.f) : 1.f;
  uint32_t sb;
  const uint32_t w = quant8(v, ts, sb);
  if (row >= rows) return;
  const int nd = SRC_BF16 ? top_k : 1;
  for (int k = 0; k < nd; ++k) {
    const size_t dst = SRC_BF16 ? static_cast<size_t>(__ldg(inv + static_cast<size_t>(row) * top_k + k)) : row;
    reinterpret_cast<uint32_t*>(codes + dst * (K / 2))[i] = w;
    if ((i & 1) == 0) scales[dst * (K / 16) + (i >> 1)] = static_cast<uint8_t>(sb);
    if (i == 0) ts_out[dst] = ts;
  }
}

// ---------------------------------------------------------------------------------------------
// routed grouped GEMM, kind::mxf4nvf4

constexpr int kW4D = 4;                            // ring depth (stages of 256 K)
constexpr int kW4ABox = 128 * 128;                 // weight codes: 128 rows x 128 bytes
constexpr int kW4BRows = kPfN;                     // activation rows per tile (MMA N, up to)
constexpr int kW4RawA = 128 * 16;                  // raw weight scales of a block and stage
constexpr int kW4RawB = kW4BRows * 16;
constexpr int kW4Atom = 512;
constexpr int kW4OffA = 0;
constexpr int kW4OffB = kW4OffA + 2 * kW4ABox;
constexpr int kW4OffRawA = kW4OffB + kW4BRows * 128;
constexpr int kW4OffRawB = kW4OffRawA + 2 * kW4RawA;
constexpr int kW4OffAtom = kW4OffRawB + kW4RawB;   // atoms: block 0 (K-steps 0..3), block 1, activations
constexpr int kW4Stage = kW4OffAtom + 12 * kW4Atom;
static_assert(kW4Stage % 1024 == 0 && kW4OffB % 1024 == 0, "128-byte swizzled operands on 1024-byte boundaries");
constexpr int kW4OffTab = kW4D * kW4Stage;
constexpr int kW4OffBar = (kW4OffTab + static_cast<int>(sizeof(TileTab)) + 7) / 8 * 8;

struct W4Bars {
  uint64_t full_a[kW4D], full_b[kW4D], sf_ready[kW4D], empty[kW4D];
  uint64_t acc_full[2], acc_empty[2], done[2];
  uint32_t tmem;
  int abort;
};
constexpr int kW4Smem = kW4OffBar + static_cast<int>(sizeof(W4Bars)) + 1024;
static_assert(kW4Smem <= 227 * 1024, "shared memory per CTA");

// tensor memory: accumulators [slot 2][block 2] x 64 columns, then per ring slot 64 scale columns:
// per weight block (the MMA warp that issues it) 16 of the block's scales (4 K-steps x 4) and 16 of
// the activations'
constexpr int kW4Threads = 448;
constexpr uint32_t kW4ColSf = 256;
constexpr uint32_t kW4SfSlot = 64;
static_assert(kW4ColSf + kW4D * kW4SfSlot <= 512, "tensor-memory columns");

template <int PHASE>
struct W4Geom;
template <>
struct W4Geom<kPhaseGateUp> {
  static constexpr int S = kH / 256, RP = kI / 128;
  __device__ static int row(int w, int rp, int b) { return w * 2 * kI + b * kI + rp * 128; }
};
template <>
struct W4Geom<kPhaseDown> {
  static constexpr int S = kI / 256, RP = kH / 256;
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

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int PHASE>
__global__ void __launch_bounds__(kW4Threads, 1) w4a4_kernel(const __grid_constant__ PrefillParams p) {
  using G = W4Geom<PHASE>;
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
      mbar_init(&bb.sf_ready[i], 2);
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
  if (warp == 0) build_tiles(tt, p, G::RP);
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
    // ---- weight codes and raw scales
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at(tt, t);
        const int r0 = G::row(tl.w, tl.rp, 0), r1 = G::row(tl.w, tl.rp, 1);
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kW4D;
          if (it >= kW4D && !pf_wait(&bb.empty[slot], ((it / kW4D) - 1) & 1, abort, p.err)) break;
          uint8_t* st = sm + slot * kW4Stage;
          mbar_arrive_expect_tx(&bb.full_a[slot], 2 * kW4ABox + 2 * kW4RawA);
          tma_2d(st + kW4OffA, &p.tm_codes, s * 128, r0, &bb.full_a[slot]);
          tma_2d(st + kW4OffA + kW4ABox, &p.tm_codes, s * 128, r1, &bb.full_a[slot]);
          tma_2d(st + kW4OffRawA, &p.tm_sc, s * 16, r0, &bb.full_a[slot]);
          tma_2d(st + kW4OffRawA + kW4RawA, &p.tm_sc, s * 16, r1, &bb.full_a[slot]);
        }
      }
      for (int j = max(it - kW4D, 0); j < it; ++j) pf_wait(&bb.full_a[j % kW4D], (j / kW4D) & 1, abort, p.err);
    }
  } else if (warp == 3) {
    // ---- activation codes and raw scales: the chunk's rows rounded up to 16
    if (lane == 0) {
      pdl_wait();
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at(tt, t);
        const int nbox = (tl.n + 15) >> 4;
        bool ok = true;
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kW4D;
          if (it >= kW4D && !pf_wait(&bb.empty[slot], ((it / kW4D) - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = sm + slot * kW4Stage;
          mbar_arrive_expect_tx(&bb.full_b[slot], nbox * (16 * 128 + 16 * 16));
          for (int q = 0; q < nbox; ++q) {
            tma_2d(st + kW4OffB + q * 2048, &p.tm_act, s * 128, tl.row0 + 16 * q, &bb.full_b[slot]);
            tma_2d(st + kW4OffRawB + q * 256, &p.tm_act_sc, s * 16, tl.row0 + 16 * q, &bb.full_b[slot]);
          }
        }
        if (!ok) break;
      }
      for (int j = max(it - kW4D, 0); j < it; ++j) pf_wait(&bb.full_b[j % kW4D], (j / kW4D) & 1, abort, p.err);
    }
  } else if (warp == 2 || warp == 13) {
    // ---- raw scales -> MMA scale atoms (lane = m0); warp 2: block 0 and activations, warp 13: block 1
    const int b_lo = warp == 2 ? 0 : 1;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      bool ok = true;
      for (int s = 0; s < G::S; ++s, ++it) {
        const int slot = it % kW4D;
        if (!pf_wait_all(&bb.full_a[slot], (it / kW4D) & 1, abort, p.err) ||
            !pf_wait_all(&bb.full_b[slot], (it / kW4D) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        uint8_t* st = sm + slot * kW4Stage;
#pragma unroll
        for (int bi = 0; bi < 2; ++bi) {        // (weight block 0, activations) or weight block 1
          const int b = bi == 0 ? b_lo : 2;
          if (b_lo == 1 && bi == 1) break;
          const uint8_t* raw = b < 2 ? st + kW4OffRawA + b * kW4RawA : st + kW4OffRawB;
          const int nm1 = b < 2 ? 4 : kW4BRows / 32;
          uint4 r[4];
#pragma unroll
          for (int m1 = 0; m1 < 4; ++m1)
            r[m1] = m1 < nm1 ? *reinterpret_cast<const uint4*>(raw + (lane + 32 * m1) * 16) : make_uint4(0, 0, 0, 0);
          uint8_t* atom = st + kW4OffAtom + b * 4 * kW4Atom + lane * 16;
          *reinterpret_cast<uint4*>(atom + 0 * kW4Atom) = make_uint4(r[0].x, r[1].x, r[2].x, r[3].x);
          *reinterpret_cast<uint4*>(atom + 1 * kW4Atom) = make_uint4(r[0].y, r[1].y, r[2].y, r[3].y);
          *reinterpret_cast<uint4*>(atom + 2 * kW4Atom) = make_uint4(r[0].z, r[1].z, r[2].z, r[3].z);
          *reinterpret_cast<uint4*>(atom + 3 * kW4Atom) = make_uint4(r[0].w, r[1].w, r[2].w, r[3].w);
        }
        fence_proxy_async_smem();               // the atoms are read by tcgen05.cp (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&bb.sf_ready[slot]);
      }
      if (!ok) break;
    }
  } else if (warp == 1 || warp == 12) {
    // ---- scale copies and MMA issue for one weight block (uniform control flow; an elected lane issues)
    const int b = warp == 1 ? 0 : 1;
    int it = 0, ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
      const PfTile tl = tile_at(tt, t);
      const uint32_t idesc = idesc_mxf4nvf4((tl.n + 15) & ~15);
      const int as = ti & 1;
      if (ti >= 2 && !pf_wait_all(&bb.acc_empty[as], ((ti >> 1) - 1) & 1, abort, p.err)) break;
      tc_fence_after();
      const uint32_t d = tmem + as * 128 + b * 64;
      for (int s = 0; s < G::S; ++s, ++it) {
        const int slot = it % kW4D;
        if (!pf_wait_all(&bb.sf_ready[slot], (it / kW4D) & 1, abort, p.err) ||
            !pf_wait_all(&bb.full_a[slot], (it / kW4D) & 1, abort, p.err) ||
            !pf_wait_all(&bb.full_b[slot], (it / kW4D) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(sm + slot * kW4Stage);
        const uint32_t sfa = tmem + kW4ColSf + slot * kW4SfSlot + b * 32, sfb = sfa + 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tc_cp_atom_w(sfa + j * 4, sdesc_atom(st + kW4OffAtom + (b * 4 + j) * kW4Atom));
          tc_cp_atom_w(sfb + j * 4, sdesc_atom(st + kW4OffAtom + (2 * 4 + j) * kW4Atom));
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
    // groups 2i + k
    const int q = warp & 3, r = 32 * q + lane, k = (warp - 4) >> 2;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    pdl_wait();                                    // the activation tensor scales are the previous kernel's output
    int ti = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++ti) {
      const PfTile tl = tile_at(tt, t);
      const int as = ti & 1;
      // the tile's scales are loaded before the wait for its accumulators: the weight tensor scales
      // and one activation tensor scale per column (column c in lane c % 32 of ts_lo / ts_hi)
      float tw0, tw1;
      if constexpr (PHASE == kPhaseGateUp) {
        tw0 = __ldg(p.tscale + 2 * tl.w);
        tw1 = __ldg(p.tscale + 2 * tl.w + 1);
      } else {
        tw0 = tw1 = __ldg(p.tscale + tl.w);
      }
      const float ts_lo = lane < tl.n ? __ldg(p.act_ts + tl.row0 + lane) : 0.f;
      const float ts_hi = lane + 32 < tl.n ? __ldg(p.act_ts + tl.row0 + 32 + lane) : 0.f;
      if (!pf_wait_all(&bb.acc_full[as], (ti >> 1) & 1, abort, p.err)) break;
      tc_fence_after();
      const uint32_t dbase = lane_base + as * 128;
      for (int j0 = 16 * k; j0 < tl.n; j0 += 32) {
        uint32_t d0[16], d1[16];
        tc_ld16(dbase + j0, d0);
        tc_ld16(dbase + 64 + j0, d1);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float ta = __shfl_sync(kAll, j0 < 32 ? ts_lo : ts_hi, (j0 + c) & 31);
          if (j0 + c < tl.n) {
            const size_t row = static_cast<size_t>(tl.row0 + j0 + c);
            const float v0 = __uint_as_float(d0[c]) * (tw0 * ta), v1 = __uint_as_float(d1[c]) * (tw1 * ta);
            if constexpr (PHASE == kPhaseGateUp) {
              p.h32[row * kI + tl.rp * 128 + r] = silu_fast(v0) * v1;
            } else {
              p.o[row * kH + tl.rp * 256 + r] = __float2half_rn(v0);
              p.o[row * kH + tl.rp * 256 + 128 + r] = __float2half_rn(v1);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bb.acc_empty[as]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

template <typename Kern>
cudaError_t launch_pdl(Kern kernel, int grid, int threads, int smem, bool pdl, cudaStream_t s, const PrefillParams& p) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace

cudaError_t launch_act_quant_x(const uint16_t* x, int T, int K, const int* inv, uint8_t* codes, uint8_t* scales,
                               float* ts, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  act_quant_kernel<kH, true><<<T, 256, 0, s>>>(x, T, K, inv, codes, scales, ts);
  return cudaGetLastError();
}

cudaError_t launch_act_quant_h(const float* h, int P, uint8_t* codes, uint8_t* scales, float* ts, bool pdl,
                               cudaStream_t s) {
  if (P <= 0) return cudaSuccess;
  constexpr int kRows = 256 / (kI / 8);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((P + kRows - 1) / kRows);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<kI, false>, static_cast<const void*>(h), P, 1,
                            static_cast<const int*>(nullptr), codes, scales, ts);
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
  return phase == kPhaseGateUp ? launch_pdl(w4a4_kernel<kPhaseGateUp>, n_sm, kW4Threads, kW4Smem, pdl, s, p)
                               : launch_pdl(w4a4_kernel<kPhaseDown>, n_sm, kW4Threads, kW4Smem, pdl, s, p);
}

}  // namespace flint
