// Expert projections for large token counts (prefill): grouped GEMMs on the fifth-generation tensor
// cores (tcgen05.mma, fp32 accumulators in tensor memory).
//
// Routed experts (pf_routed_kernel). The permuted rows of one expert are its tokens; a tile is
// (expert, a chunk of up to 64 of those rows, a pair of 128-row weight blocks): for gate|up the
// gate rows [128r, 128r+128) and the matching up rows, for down the output rows [256r, 256r+128)
// and [256r+128, 256r+256). One persistent CTA per SM walks the tiles; its warps specialise:
//   warp 0       TMA copies of the 4-bit codes, 128 K per stage, into a shared-memory ring
//   warp 3       TMA copies of the chunk's activation rows (fp16, stored per permuted row so that
//                an expert's rows are contiguous; 128-byte swizzled K-major, 16-row boxes) into a ring
//   warps 4..    dequantisation (8 or 16 warps): a thread owns one weight row of one block and both
//                64-code halves of the stage, or one of them, turns those codes into exact fp16
//                (int4: code x bf16 group scale; NVFP4: E2M1 x E4M3) and writes them to tensor
//                memory with tcgen05.st, where the MMA reads its A operand. A in tensor memory costs
//                no shared-memory bandwidth, which a 128 x 48 MMA with A in shared memory would
//                exhaust.
//   warps 1, 2   MMA issue, one warp per block with an elected lane issuing (an MMA instruction
//                takes ~45 cycles to issue, so two issuers keep N = 48 tiles near the tensor-core
//                rate); D[128 x N] per block, double-buffered
//   last 4 warps epilogue: gate|up -> h = silu(g) u, int4: rotated per 128-segment by the Hadamard
//                butterfly, stored fp16 in the order of the down operand; down -> o in fp16.
// Every dependency is an mbarrier: TMA transaction counts, tcgen05.commit arrivals and thread
// arrivals; every wait is bounded and sets a timeout bit on expiry. The routed down kernel is a
// programmatic dependent of the gate|up kernel: its code copies start as soon as it has an SM, its
// activation copies after griddepcontrol.wait.
//
// The shared expert (pf_shared_kernel) is a dense bf16 GEMM of the same shape of pipeline with the
// weights and activations brought by TMA in the 128-byte swizzled layout and read by the MMA from
// shared memory.
#include "common.cuh"
#include "kernels.cuh"
#include "tc.cuh"

namespace flint {

namespace {

constexpr int kPfSK = 128;                   // K per pipeline stage
constexpr int kPfDA = 6;                     // code ring depth
constexpr int kPfDB = 6;                     // activation ring depth
constexpr int kPfCodeStage = 2 * 128 * kPfSK / 2;    // 16 KB: two blocks of 128 rows x 64 bytes
constexpr int kPfActChunk = kPfN * 128;              // 64 K of every row, 128-byte swizzled
constexpr int kPfActStage = 2 * kPfActChunk;         // 16 KB
constexpr int kSlabPitch = 132;              // floats per token row of the epilogue's transpose slab
// Dequantisation warps: 4 lane quarters x 2 blocks, x 2 halves of the stage when there are 16. The
// int4 gate|up tiles run fastest with 8 (two halves per thread), the others with 16 (measured).
template <int FMT, int PHASE>
struct PfRoles {
  static constexpr int kDq = (FMT == kInt4 && PHASE == kPhaseGateUp) ? 8 : 16;
  static constexpr int kHalves = 16 / kDq;          // stage halves per dequantisation thread
  static constexpr int kThreads = 32 * (4 + kDq + 4);
};

// tensor-memory columns: two accumulator slots of (D0 | D1) x 64 columns, then two A stages of two
// blocks x 64 columns (128 fp16 of K)
constexpr uint32_t kColD1 = 64;
constexpr uint32_t kColSlot = 128;
constexpr uint32_t kColA = 256;

template <int PHASE>
struct PfGeom;
template <>
struct PfGeom<kPhaseGateUp> {
  static constexpr int K = kH, S = kH / kPfSK, RP = kI / 128;
  // first weight row of block b of a tile
  __device__ static int row(int e, int rp, int b) { return e * 2 * kI + b * kI + rp * 128; }
};
template <>
struct PfGeom<kPhaseDown> {
  static constexpr int K = kI, S = kI / kPfSK, RP = kH / 256;
  __device__ static int row(int e, int rp, int b) { return e * kH + rp * 256 + b * 128; }
};

// shared-memory layout of the routed kernel (offsets from a 1024-byte aligned base)
constexpr int kOffAct = 0;
constexpr int kOffCode = kOffAct + kPfDB * kPfActStage;
constexpr int kOffSlab = kOffCode + kPfDA * kPfCodeStage;
constexpr int kOffTab = kOffSlab + 32 * kSlabPitch * 4;
constexpr int kOffBar = (kOffTab + static_cast<int>(sizeof(TileTab)) + 7) / 8 * 8;

struct PfBars {
  uint64_t code_full[kPfDA], code_empty[kPfDA];
  uint64_t act_full[kPfDB], act_empty[kPfDB];
  uint64_t a_full[2][2], a_empty[2][2];       // [A stage in tensor memory][block]
  uint64_t acc_full[2][2], acc_empty[2];       // [accumulator slot][block]
  uint64_t done[2];
  uint32_t tmem;
  int abort;
};
constexpr int kPfSmem = kOffBar + static_cast<int>(sizeof(PfBars)) + 1024;   // + alignment slack
static_assert(kPfSmem <= 227 * 1024, "shared memory per CTA");

// int4 scale (bf16) -> fp16 pair; flags scales whose products with the codes fp16 cannot hold exactly
__device__ __forceinline__ uint32_t scale_half2(uint32_t bf16_bits, bool& bad) {
  const float s = bf16_bits_to_f32(static_cast<uint16_t>(bf16_bits));
  const float a = fabsf(s);
  bad |= (a > 8188.f) || (a != 0.f && a < 6.103515625e-05f);
  return pack_half2(s, s);
}

// Turns 64 codes (8 words) of one row into 32 fp16 pairs: 32 tensor-memory columns of the row.
// int4: word w gives columns 4w..4w+3 = pairs (n0,n4),(n1,n5),(n2,n6),(n3,n7) of its eight codes
// (the order the activation operand is stored in). NVFP4: natural order; `s_blk` holds the four
// E4M3 scales of the 16-code blocks.
template <int FMT>
__device__ __forceinline__ void dequant_half(uint32_t (&v)[32], const uint4& wa, const uint4& wb, uint32_t s_int4,
                                             uint32_t s_blk) {
  const uint32_t words[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if constexpr (FMT == kInt4) {
      uint32_t pr[4];
      int4x8_to_half2x4(words[k], pr);
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * k + j] = hmul2_u32(pr[j], s_int4);
    } else {
      const uint32_t h = e4m3_to_half_bits((s_blk >> (8 * (k >> 1))) & 0xFFu);
      const uint32_t s2 = h | (h << 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * k + j] = hmul2_u32(e2m1x2_to_half2(words[k] >> (8 * j)), s2);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// routed grouped GEMM

template <int FMT, int PHASE>
__global__ void __launch_bounds__(PfRoles<FMT, PHASE>::kThreads, 1) pf_routed_kernel(const __grid_constant__ PrefillParams p) {
  using G = PfGeom<PHASE>;
  using R = PfRoles<FMT, PHASE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  TileTab& tt = *reinterpret_cast<TileTab*>(sm + kOffTab);
  PfBars& bb = *reinterpret_cast<PfBars*>(sm + kOffBar);
  float* slab = reinterpret_cast<float*>(sm + kOffSlab);
  volatile int* abort = &bb.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPfDA; ++i) {
      mbar_init(&bb.code_full[i], 1);
      mbar_init(&bb.code_empty[i], R::kDq);
    }
    for (int i = 0; i < kPfDB; ++i) {
      mbar_init(&bb.act_full[i], 1);
      mbar_init(&bb.act_empty[i], 2);
    }
    for (int t = 0; t < 2; ++t)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bb.a_full[t][b], R::kDq / 2);
        mbar_init(&bb.a_empty[t][b], 1);
      }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bb.acc_full[a][0], 1);
      mbar_init(&bb.acc_full[a][1], 1);
      mbar_init(&bb.acc_empty[a], 4);
    }
    mbar_init(&bb.done[0], 1);
    mbar_init(&bb.done[1], 1);
    bb.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) build_tiles<false>(tt, p, G::RP);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&bb.tmem)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bb.tmem;
  const int total = tt.total;
  pdl_trigger();   // the next kernel's CTAs take the SMs this grid leaves (it is resident in full)

  if (warp == 0) {
    // ---- codes: two TMA boxes (128 rows x 64 bytes) per stage (read once: evicted first from L2)
    int it = 0;
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at<false>(tt, t);
        const int r0 = G::row(tl.w, tl.rp, 0), r1 = G::row(tl.w, tl.rp, 1);
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kPfDA;
          if (it >= kPfDA && !pf_wait(&bb.code_empty[slot], ((it / kPfDA) - 1) & 1, abort, p.err)) break;
          uint8_t* st = sm + kOffCode + slot * kPfCodeStage;
          mbar_arrive_expect_tx(&bb.code_full[slot], kPfCodeStage);
          tma_2d_hint(st, &p.tm_codes, s * (kPfSK / 8), r0, &bb.code_full[slot], pol);
          tma_2d_hint(st + kPfCodeStage / 2, &p.tm_codes, s * (kPfSK / 8), r1, &bb.code_full[slot], pol);
        }
      }
      // no copy may still be in flight when the CTA exits
      for (int j = max(it - kPfDA, 0); j < it; ++j) pf_wait(&bb.code_full[j % kPfDA], (j / kPfDA) & 1, abort, p.err);
    }
  } else if (warp == 3) {
    // ---- activations: the chunk's rows are contiguous (permuted order); per stage and 64-K half, the
    // chunk's rows rounded up to 16 in boxes of 16 rows x 64 fp16 (128-byte swizzled, 2 KB each);
    // rows past the chunk only feed unused accumulator columns
    if (lane == 0) {
      pdl_wait();     // the activation rows are the previous kernel's output
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const PfTile tl = tile_at<false>(tt, t);
        const int nbox = (tl.n + 15) >> 4;
        bool ok = true;
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % kPfDB;
          if (it >= kPfDB && !pf_wait(&bb.act_empty[slot], ((it / kPfDB) - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = sm + kOffAct + slot * kPfActStage;
          mbar_arrive_expect_tx(&bb.act_full[slot], nbox * 2 * 2048);
          for (int q = 0; q < nbox; ++q) {
            tma_2d(st + q * 2048, &p.tm_act, s * kPfSK, tl.row0 + 16 * q, &bb.act_full[slot]);
            tma_2d(st + kPfActChunk + q * 2048, &p.tm_act, s * kPfSK + 64, tl.row0 + 16 * q, &bb.act_full[slot]);
          }
        }
        if (!ok) break;
      }
      for (int j = max(it - kPfDB, 0); j < it; ++j) pf_wait(&bb.act_full[j % kPfDB], (j / kPfDB) & 1, abort, p.err);
    }
  } else if (warp == 1 || warp == 2) {
    // ---- MMA issue, one warp per block (uniform control flow; an elected lane issues)
    const int b = warp - 1;
    int it = 0, ti = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++ti) {
      const PfTile tl = tile_at<false>(tt, t);
      const int npad = (tl.n + 15) & ~15;
      const uint32_t idesc = idesc_m128(npad, false);
      const int as = ti & 1;
      const uint32_t d = tmem + as * kColSlot + b * kColD1;
      if (ti >= 2 && !pf_wait_all(&bb.acc_empty[as], ((ti >> 1) - 1) & 1, abort, p.err)) break;
      tc_fence_after();
      for (int s = 0; s < G::S; ++s, ++it) {
        const int ts = it & 1, bs = it % kPfDB;
        if (!pf_wait_all(&bb.a_full[ts][b], (it >> 1) & 1, abort, p.err) ||
            !pf_wait_all(&bb.act_full[bs], (it / kPfDB) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = tmem + kColA + ts * 128 + b * 64;
        const uint32_t b0 = smem_u32(sm + kOffAct + bs * kPfActStage);
#pragma unroll
        for (int ks = 0; ks < kPfSK / 16; ++ks)
          tc_mma_ta_w(d, a0 + ks * 8, sdesc_sw128(b0 + (ks >> 2) * kPfActChunk + (ks & 3) * 32), idesc,
                      (s | ks) ? 1u : 0u);
        tc_commit_w(&bb.a_empty[ts][b]);
        tc_commit_w(&bb.act_empty[bs]);
      }
      if (ok) tc_commit_w(&bb.acc_full[as][b]);
    }
    tc_commit_w(&bb.done[b]);                     // every MMA of this warp has completed
    pf_wait_all(&bb.done[b], 0, abort, p.err);
  } else if (warp >= 4 && warp < 4 + R::kDq) {
    // ---- dequantisation into tensor memory
    const int b = ((warp - 4) >> 2) & 1, h0 = (warp - 4) >> 3, q = warp & 3;   // h0: first half
    const int r = 32 * q + lane;
    const int swz = (lane >> 1) & 3;               // 64-byte swizzle of the code rows (row r at r*64)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    // Scales are fetched ahead: int4 all of the row's group scales one tile ahead; NVFP4 the 16 E4M3
    // block scales of a stage pair one pair ahead.
    constexpr int kSc4 = FMT == kInt4 ? G::S / 2 : 1;
    uint32_t sc_next[kSc4];
    uint4 fp_next = make_uint4(0, 0, 0, 0);
    auto load_int4 = [&](int row) {
      const uint32_t* s32 = reinterpret_cast<const uint32_t*>(p.scales) + static_cast<size_t>(row) * (G::S / 2);
#pragma unroll
      for (int k = 0; k < kSc4; ++k) sc_next[k] = __ldg(s32 + k);
    };
    auto load_fp4 = [&](int row, int pair) {
      fp_next = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.scales) +
                                                     static_cast<size_t>(row) * (G::K / 16) + pair * 16));
    };
    int t = blockIdx.x;
    int row = 0;
    if (t < total) {
      const PfTile tl = tile_at<false>(tt, t);
      row = G::row(tl.w, tl.rp, b) + r;
      if constexpr (FMT == kInt4) load_int4(row);
      else load_fp4(row, 0);
    }
    int it = 0;
    bool bad = false;
    while (t < total && !*abort) {
      const int t_next = t + gridDim.x;
      int row_next = -1;
      if (t_next < total) {
        const PfTile tn = tile_at<false>(tt, t_next);
        row_next = G::row(tn.w, tn.rp, b) + r;
      }
      uint32_t sc[kSc4];                         // consumed from sc[0], shifted down every 2 stages
#pragma unroll
      for (int k = 0; k < kSc4; ++k) sc[k] = sc_next[k];
      if constexpr (FMT == kInt4) {
        if (row_next >= 0) load_int4(row_next);
      }
      uint4 fp_cur = make_uint4(0, 0, 0, 0);
      bool ok = true;
      for (int s = 0; s < G::S; ++s, ++it) {
        const int slot = it % kPfDA, ts = it & 1;
        uint2 s_fp4 = make_uint2(0, 0);
        if constexpr (FMT == kNvfp4) {
          if ((s & 1) == 0) {
            fp_cur = fp_next;
            if (s + 2 < G::S) load_fp4(row, (s + 2) >> 1);
            else if (row_next >= 0) load_fp4(row_next, 0);
          }
          s_fp4 = (s & 1) ? make_uint2(fp_cur.z, fp_cur.w) : make_uint2(fp_cur.x, fp_cur.y);
        }
        if (!pf_wait_all(&bb.code_full[slot], (it / kPfDA) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        const uint8_t* src = sm + kOffCode + slot * kPfCodeStage + b * (kPfCodeStage / 2) + r * (kPfSK / 2);
        uint4 w[2 * R::kHalves];                  // the row's 16-byte chunks of its halves
#pragma unroll
        for (int k = 0; k < 2 * R::kHalves; ++k) w[k] = *reinterpret_cast<const uint4*>(src + (((2 * h0 + k) ^ swz) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&bb.code_empty[slot]);
        uint32_t s_int4 = 0;
        if constexpr (FMT == kInt4) {
          s_int4 = scale_half2((sc[0] >> (16 * (s & 1))) & 0xFFFFu, bad);
          if (s & 1) {
#pragma unroll
            for (int k = 0; k + 1 < kSc4; ++k) sc[k] = sc[k + 1];
          }
        }
        // the first half's arithmetic runs before the tensor-memory stage is free
        uint32_t v[32];
        dequant_half<FMT>(v, w[0], w[1], s_int4, h0 ? s_fp4.y : s_fp4.x);
        if (it >= 2 && !pf_wait_all(&bb.a_empty[ts][b], ((it >> 1) - 1) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = lane_base + kColA + ts * 128 + b * 64 + h0 * 32;
        tc_st32(ta, v);
        if constexpr (R::kHalves == 2) {
          dequant_half<FMT>(v, w[2], w[3], s_int4, s_fp4.y);
          tc_st32(ta + 32, v);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bb.a_full[ts][b]);
      }
      if (!ok) break;
      t = t_next;
      row = row_next;
    }
    if (bad) atomicOr(p.err, kErrRange);
  } else if (warp >= 4 + R::kDq) {
    // ---- epilogue
    const int q = warp & 3, r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    int ti = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++ti) {
      const PfTile tl = tile_at<false>(tt, t);
      const int as = ti & 1;
      if (!pf_wait_all(&bb.acc_full[as][0], (ti >> 1) & 1, abort, p.err) ||
          !pf_wait_all(&bb.acc_full[as][1], (ti >> 1) & 1, abort, p.err))
        break;
      tc_fence_after();
      const uint32_t dbase = lane_base + as * kColSlot;
      if constexpr (PHASE == kPhaseGateUp) {
        float tsg = 1.f, tsu = 1.f;
        if (p.tscale) {
          tsg = p.tscale[2 * tl.w];
          tsu = p.tscale[2 * tl.w + 1];
        }
        for (int j0 = 0; j0 < tl.n; j0 += 32) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (j0 + 16 * hf < tl.n) {
              uint32_t g[16], u[16];
              tc_ld16(dbase + j0 + 16 * hf, g);
              tc_ld16(dbase + kColD1 + j0 + 16 * hf, u);
              tc_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float gv = __uint_as_float(g[c]) * tsg, uv = __uint_as_float(u[c]) * tsu;
                slab[(16 * hf + c) * kSlabPitch + r] = silu_fast(gv) * uv;
              }
            }
          }
          named_bar_sync(1, 128);
          for (int jj = 8 * q; jj < 8 * q + 8; ++jj) {
            if (j0 + jj >= tl.n) break;
            const float4 hv = *reinterpret_cast<const float4*>(slab + jj * kSlabPitch + 4 * lane);
            float v[4] = {hv.x, hv.y, hv.z, hv.w};
            if constexpr (FMT == kInt4) fwht128_warp(v);
            store_seg_half(p.hq + static_cast<size_t>(tl.row0 + j0 + jj) * kI + tl.rp * 128, v, FMT == kInt4);
          }
          named_bar_sync(1, 128);
        }
      } else {
        const float ts = p.tscale ? p.tscale[tl.w] : 1.f;
        for (int j0 = 0; j0 < tl.n; j0 += 16) {
          uint32_t d0[16], d1[16];
          tc_ld16(dbase + j0, d0);
          tc_ld16(dbase + kColD1 + j0, d1);
          tc_wait_ld();
          __half* orow = p.o + static_cast<size_t>(tl.row0 + j0) * kH + tl.rp * 256 + r;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            if (j0 + c < tl.n) {
              orow[static_cast<size_t>(c) * kH] = __float2half_rn(__uint_as_float(d0[c]) * ts);
              orow[static_cast<size_t>(c) * kH + 128] = __float2half_rn(__uint_as_float(d1[c]) * ts);
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

// ---------------------------------------------------------------------------------------------
// shared expert: dense bf16 GEMM, operands by TMA

constexpr int kShThreads = 256;
constexpr uint32_t kShColD1 = 128;                   // D1 after the 128 columns of D0
constexpr int kShBox = 128 * 128;                    // 128 rows x 64 bf16, 128-byte swizzled

template <int PHASE>
struct ShGeom;
template <>
struct ShGeom<kPhaseGateUp> {
  static constexpr int S = kH / 64, RP = kIs / 128, NB = 1, D = 4;
  __device__ static int row(int rp, int b) { return b * kIs + rp * 128; }
};
template <>
struct ShGeom<kPhaseDown> {
  static constexpr int S = kIs / 64, RP = kH / 256, NB = 2, D = 3;
  __device__ static int row(int rp, int b) { return rp * 256 + b * 128; }
};
// router logits: A = router rows (experts rp*256 + b*128 ..), B = x; RP = ceil(E / 256) at run time;
// K is split in kRouterSplit slices (one per tile) whose partial logits the top-k kernel sums
template <>
struct ShGeom<kPhaseRouter> {
  static constexpr int S = kH / 64 / kRouterSplit, RP = 0, NB = 1, D = 4;
  __device__ static int row(int rp, int b) { return rp * 256 + b * 128; }
};

template <int PHASE>
struct ShLayout {
  using G = ShGeom<PHASE>;
  static constexpr int kStage = (2 + G::NB) * kShBox;
  static constexpr int kOffBar = G::D * kStage;
};

struct ShBars {
  uint64_t full[4], empty[4];
  uint64_t acc_full[2], acc_empty[2], fin[2];
  uint32_t tmem;
  int abort;
};

template <int PHASE>
constexpr int sh_smem() {
  return ShLayout<PHASE>::kOffBar + static_cast<int>(sizeof(ShBars)) + 1024;
}
static_assert(sh_smem<kPhaseGateUp>() <= 227 * 1024 && sh_smem<kPhaseDown>() <= 227 * 1024 &&
                  sh_smem<kPhaseRouter>() <= 227 * 1024,
              "shared memory per CTA");

template <int PHASE>
__global__ void __launch_bounds__(kShThreads, 1) pf_shared_kernel(const __grid_constant__ PrefillParams p) {
  using G = ShGeom<PHASE>;
  using L = ShLayout<PHASE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  ShBars& bb = *reinterpret_cast<ShBars*>(sm + L::kOffBar);
  volatile int* abort = &bb.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = (p.T + 127) / 128;
  const int nrp = PHASE == kPhaseRouter ? (p.E + 255) / 256 : G::RP;
  const int total = nrp * nch * (PHASE == kPhaseRouter ? kRouterSplit : 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < G::D; ++i) {
      mbar_init(&bb.full[i], 1);
      mbar_init(&bb.empty[i], 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bb.acc_full[b], 1);
      mbar_init(&bb.acc_empty[b], 1);
      mbar_init(&bb.fin[b], 1);
    }
    bb.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(smem_u32(&bb.tmem)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bb.tmem;
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();    // a programmatic launch (shared down) reads the previous kernel's hidden pair
      int it = 0;
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const int ks = t / (nrp * nch), tr = t - ks * (nrp * nch);   // K slice (router only)
        const int rp = tr / nch, c0 = (tr - rp * nch) * 128;
        for (int s = 0; s < G::S; ++s, ++it) {
          const int slot = it % G::D;
          if (it >= G::D && !pf_wait(&bb.empty[slot], ((it / G::D) - 1) & 1, abort, p.err)) break;
          uint8_t* st = sm + slot * L::kStage;
          const int kx = (ks * G::S + s) * 64;
          mbar_arrive_expect_tx(&bb.full[slot], L::kStage);
          tma_2d(st, &p.tm_a, kx, G::row(rp, 0), &bb.full[slot]);
          tma_2d(st + kShBox, &p.tm_a, kx, G::row(rp, 1), &bb.full[slot]);
          tma_2d(st + 2 * kShBox, &p.tm_b, kx, c0, &bb.full[slot]);
          if constexpr (G::NB == 2) tma_2d(st + 3 * kShBox, &p.tm_b2, kx, c0, &bb.full[slot]);
        }
      }
      for (int j = max(it - G::D, 0); j < it; ++j) pf_wait(&bb.full[j % G::D], (j / G::D) & 1, abort, p.err);
    }
  } else if (warp == 1 || warp == 2) {
    const int b = warp - 1;                       // one warp per block; an elected lane issues
    int it = 0;
    bool ok = true;
    const uint32_t idesc = idesc_m128(128, true);
    const uint32_t d = tmem + b * kShColD1;
    for (int t = blockIdx.x, ti = 0; t < total && ok; t += gridDim.x, ++ti) {
      if (ti > 0 && !pf_wait_all(&bb.acc_empty[b], (ti - 1) & 1, abort, p.err)) break;   // D drained
      tc_fence_after();
      for (int s = 0; s < G::S; ++s, ++it) {
        const int slot = it % G::D;
        if (!pf_wait_all(&bb.full[slot], (it / G::D) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(sm + slot * L::kStage);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = sdesc_sw128(st + b * kShBox + ks * 32);
          tc_mma_ss_w(d, ad, sdesc_sw128(st + 2 * kShBox + ks * 32), idesc, (s | ks) ? 1u : 0u);
          if constexpr (G::NB == 2) tc_mma_ss_w(d, ad, sdesc_sw128(st + 3 * kShBox + ks * 32), idesc, 1u);
        }
        tc_commit_w(&bb.empty[slot]);
      }
      if (ok) tc_commit_w(&bb.acc_full[b]);
    }
    tc_commit_w(&bb.fin[b]);                      // every MMA of this warp has completed
    pf_wait_all(&bb.fin[b], 0, abort, p.err);
  } else if (warp >= 4) {
    const int q = warp & 3, r = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    for (int t = blockIdx.x, ti = 0; t < total; t += gridDim.x, ++ti) {
      const int ks = t / (nrp * nch), tr = t - ks * (nrp * nch);
      const int rp = tr / nch, c0 = (tr - rp * nch) * 128;
      const int n = min(128, p.T - c0);
      float* lg = p.logits + static_cast<size_t>(ks) * p.T * p.E;
      if (!pf_wait_all(&bb.acc_full[0], ti & 1, abort, p.err) || !pf_wait_all(&bb.acc_full[1], ti & 1, abort, p.err))
        break;
      tc_fence_after();
      for (int j0 = 0; j0 < n; j0 += 16) {
        uint32_t d0[16], d1[16];
        tc_ld16(lane_base + j0, d0);
        tc_ld16(lane_base + kShColD1 + j0, d1);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (j0 + c >= n) break;
          const size_t tok = static_cast<size_t>(c0 + j0 + c);
          if constexpr (PHASE == kPhaseRouter) {
            const int e0 = rp * 256 + r;
            if (e0 < p.E) lg[tok * p.E + e0] = __uint_as_float(d0[c]);
            if (e0 + 128 < p.E) lg[tok * p.E + e0 + 128] = __uint_as_float(d1[c]);
          } else if constexpr (PHASE == kPhaseGateUp) {
            const float hs = silu_fast(__uint_as_float(d0[c])) * __uint_as_float(d1[c]);
            const uint16_t hi = f32_to_bf16_bits(hs);
            const uint16_t lo = f32_to_bf16_bits(hs - bf16_bits_to_f32(hi));
            p.hs_hi[tok * kIs + rp * 128 + r] = hi;
            p.hs_lo[tok * kIs + rp * 128 + r] = lo;
          } else {
            p.ys[tok * kH + rp * 256 + r] = __uint_as_float(d0[c]);
            p.ys[tok * kH + rp * 256 + 128 + r] = __uint_as_float(d1[c]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      named_bar_sync(1, 128);
      if (threadIdx.x == 128) {                     // D drained: the issuers may overwrite it
        mbar_arrive(&bb.acc_empty[0]);
        mbar_arrive(&bb.acc_empty[1]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem));
}

// ---------------------------------------------------------------------------------------------
// combine: y[t][n] = bf16(routed_scale * sum_k w[t][k] * o[inv[t][k]][n] + ys[t][n]), the slots
// summed in slot order (ascending expert id) in fp32, one rounding at the end. One CTA per token,
// 8 columns per thread; the loads of all slots are issued before the sum.
template <int KMAX>
__global__ void __launch_bounds__(256) pf_combine_kernel(const __half* __restrict__ o, const float* __restrict__ ys,
                                                         const float* __restrict__ w, const int* __restrict__ inv,
                                                         int K, float routed_scale, uint16_t* __restrict__ y) {
  const int t = blockIdx.x;
  const int n = threadIdx.x * 8;
  pdl_wait();      // o is the previous kernel's output
  // every slot's row index and weight first, then all rows' loads in flight together
  int row[KMAX];
  float wk[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    row[k] = k < K ? __ldg(inv + t * K + k) : 0;
    wk[k] = k < K ? __ldg(w + t * K + k) : 0.f;
  }
  uint4 ov[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k)
    ov[k] = k < K ? __ldg(reinterpret_cast<const uint4*>(o + static_cast<size_t>(row[k]) * kH + n)) : make_uint4(0, 0, 0, 0);
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(ys + static_cast<size_t>(t) * kH + n));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(ys + static_cast<size_t>(t) * kH + n + 4));
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {                 // slot order
    if (k < K) {
      const uint32_t ow[4] = {ov[k].x, ov[k].y, ov[k].z, ov[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ow[j]));
        acc[2 * j] = fmaf(wk[k], f.x, acc[2 * j]);
        acc[2 * j + 1] = fmaf(wk[k], f.y, acc[2 * j + 1]);
      }
    }
  }
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  uint4 out;
  uint32_t* ou = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    ou[j] = pack_bf162(fmaf(routed_scale, acc[2 * j], sv[2 * j]), fmaf(routed_scale, acc[2 * j + 1], sv[2 * j + 1]));
  *reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * kH + n) = out;
}

template <typename Kern>
cudaError_t allow_smem(Kern kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_prefill_routed(const PrefillParams& p, int fmt, int phase, int n_sm, bool pdl, cudaStream_t s) {
  static bool smem_set = false;
  if (!smem_set) {
    cudaError_t e;
    if ((e = allow_smem(pf_routed_kernel<kInt4, kPhaseGateUp>, kPfSmem)) != cudaSuccess) return e;
    if ((e = allow_smem(pf_routed_kernel<kInt4, kPhaseDown>, kPfSmem)) != cudaSuccess) return e;
    if ((e = allow_smem(pf_routed_kernel<kNvfp4, kPhaseGateUp>, kPfSmem)) != cudaSuccess) return e;
    if ((e = allow_smem(pf_routed_kernel<kNvfp4, kPhaseDown>, kPfSmem)) != cudaSuccess) return e;
    smem_set = true;
  }
  if (fmt == kInt4) {
    return phase == kPhaseGateUp
               ? launch_pdl_kernel(pf_routed_kernel<kInt4, kPhaseGateUp>, n_sm, PfRoles<kInt4, kPhaseGateUp>::kThreads,
                                  kPfSmem, pdl, s, p)
               : launch_pdl_kernel(pf_routed_kernel<kInt4, kPhaseDown>, n_sm, PfRoles<kInt4, kPhaseDown>::kThreads,
                                  kPfSmem, pdl, s, p);
  } else {
    return phase == kPhaseGateUp
               ? launch_pdl_kernel(pf_routed_kernel<kNvfp4, kPhaseGateUp>, n_sm, PfRoles<kNvfp4, kPhaseGateUp>::kThreads,
                                  kPfSmem, pdl, s, p)
               : launch_pdl_kernel(pf_routed_kernel<kNvfp4, kPhaseDown>, n_sm, PfRoles<kNvfp4, kPhaseDown>::kThreads,
                                  kPfSmem, pdl, s, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_prefill_shared(const PrefillParams& p, int phase, int n_sm, cudaStream_t s, bool pdl) {
  static bool smem_set = false;
  if (!smem_set) {
    cudaError_t e;
    if ((e = allow_smem(pf_shared_kernel<kPhaseGateUp>, sh_smem<kPhaseGateUp>())) != cudaSuccess) return e;
    if ((e = allow_smem(pf_shared_kernel<kPhaseDown>, sh_smem<kPhaseDown>())) != cudaSuccess) return e;
    if ((e = allow_smem(pf_shared_kernel<kPhaseRouter>, sh_smem<kPhaseRouter>())) != cudaSuccess) return e;
    smem_set = true;
  }
  const int rp = phase == kPhaseGateUp ? ShGeom<kPhaseGateUp>::RP
                 : phase == kPhaseDown ? ShGeom<kPhaseDown>::RP
                                       : (p.E + 255) / 256 * kRouterSplit;
  const int tiles = rp * ((p.T + 127) / 128);
  const int grid = tiles < n_sm ? tiles : n_sm;
  if (phase == kPhaseGateUp) return launch_pdl_kernel(pf_shared_kernel<kPhaseGateUp>, grid, kShThreads, sh_smem<kPhaseGateUp>(), pdl, s, p);
  if (phase == kPhaseDown) return launch_pdl_kernel(pf_shared_kernel<kPhaseDown>, grid, kShThreads, sh_smem<kPhaseDown>(), pdl, s, p);
  return launch_pdl_kernel(pf_shared_kernel<kPhaseRouter>, grid, kShThreads, sh_smem<kPhaseRouter>(), pdl, s, p);
}

cudaError_t launch_prefill_combine(const __half* o, const float* ys, const float* w, const int* inv, int T, int K,
                                   float routed_scale, uint16_t* y, bool pdl, cudaStream_t s) {
  static_assert(kH == 256 * 8, "one CTA of 256 threads x 8 columns per token");
  return launch_pdl_kernel(pf_combine_kernel<kMaxTopK>, T, 256, 0, pdl, s, o, ys, w, inv, K, routed_scale, y);
}

}  // namespace flint
