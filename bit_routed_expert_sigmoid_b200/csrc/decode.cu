// Whole-layer forward for small token counts (T <= 8): ONE persistent kernel, one CTA per SM,
// launched cooperatively so that every CTA is resident at once.
//
// A decode forward streams 23-92 MB of weights through the chain router -> selection -> gate|up ->
// down -> combine. Each arrow that needs data from every SM is a grid barrier inside the kernel
// (an arrival counter and a generation word in global memory, one bounded wait per CTA), not a
// kernel boundary, and every SM keeps weight copies in flight across it.
//
//   phase A  no dependencies (12 warps per CTA). Warps 4-7 compute the router logits (a K quarter
//            each, x staged by one bulk copy) and the routed experts' activation operand (a warp per
//            128-segment of a token); warps 0-3 start streaming the shared expert's gate|up tiles at
//            once; one thread asks L2 for the shared expert's down rows.
//   barrier 1
//   phase B  every CTA selects the top-k of every token from the logits (a warp per token) and
//            builds the routing tables in its own shared memory; then the routed gate|up tiles of
//            the active experts (8 gate + 8 up rows, all of K, per tile). The warp that finishes
//            the last of the 16 tiles of a 128-segment of h turns that segment into the down
//            operand (last-arriver counter; nobody waits for it). Before the barrier every warp
//            already requests its first down stages.
//   barrier 2
//   phase C  CTA c owns output rows [2048c/G, 2048(c+1)/G) of y (13-14 rows on 148 SMs), so the
//            combine needs no other CTA: it streams those rows of every active expert's down
//            matrix and of the shared expert's down matrix (eight K slices), keeps the partial
//            results in shared memory and sums them in a fixed order:
//            y = bf16(routed_scale * sum_k w_k o_k + ys).
//
// Arithmetic. Decode is bound by HBM, and at 6.5 TB/s an SM may spend only a few instructions per
// weight byte, so the cost of turning 4-bit codes into MMA operands decides the speed.
//   int4     codes become exact int8 values 16c with two bit operations per four codes, and run on
//            the integer tensor cores (m16n8k32, s8 x s8/u8 -> s32) against the activation held as a
//            16-bit fixed-point number per 128-segment, split into a signed high and an unsigned
//            low byte. Products and sums are exact integers; the group scale and the segment's
//            power-of-two unit multiply the int32 sum once per group in fp32. The only rounding
//            before the fp32 accumulation is that of the activation to 2^-14 of its segment's
//            largest power of two, finer than fp16's 2^-11 per element.
//   NVFP4    codes are converted by the hardware E2M1 -> fp16 conversion and multiplied by their
//            E4M3 block scale in fp16 (exact), then fp16 MMA with fp32 accumulation.
//   bf16     (shared expert) bf16 MMA with fp32 accumulation.
// Every wait is bounded: the mbarrier waits on a warp's own copies and the two grid barriers give
// up after 1 s of %globaltimer and set the timeout bit of the error word; a grid wait that gives up
// also sets an abort word that makes every later grid wait of the forward return at once, so a
// forward always ends.
#include "frag.cuh"
#include "kernels.cuh"

namespace flint {

namespace {

#ifndef FLINT_WAIT_NS
#define FLINT_WAIT_NS 1000000000ull          // 1 s
#endif
constexpr uint64_t kWaitNs = FLINT_WAIT_NS;
constexpr unsigned kFull = 0xFFFFFFFFu;

constexpr int kRouteWarp0 = 4;               // warps 4..7: router rows, operand
constexpr int kRouteWarps = 4;               // one per K quarter of the router rows
constexpr int kRouteThreads = kRouteWarps * 32;
constexpr int kTabWarps = kMaxE / 32;        // the routing tables take one thread per expert
constexpr int kBarRoute = 1;                 // named barrier of the routing warps
constexpr int kMaxRowsPerCta = 16;           // phase C rows of y per CTA (one MMA tile)
constexpr int kShDnSlices = kIs / kGroup;    // shared down K slices of 128 (8)

// Asks L2 to fetch [ptr, ptr + bytes) from HBM (a hint; no completion to wait for).
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

// Arrival of the calling thread on a counter with acquire-release semantics at GPU scope; returns
// the previous value.
__device__ __forceinline__ int atom_add_acq_rel(int* ctr, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(ctr), "r"(v) : "memory");
  return old;
}

// A warp's arrivals on segment counters whose results are examined only at the end of the phase:
// the warp barrier orders every lane's earlier global writes before lane 0's acquire-release add,
// and the add's return value is not read until settle(), so no tile waits for an atomic's round
// trip. Up to four arrivals are held (a warp has at most four routed gate|up tiles at the shapes
// this kernel runs; a fifth settles the first four early). settle() calls finish(counter index) for
// each counter this warp's arrival completed (the returned value was target - 1: the warp was the
// last arriver, and lane 0's acquire precedes every lane's later reads).
struct PendingArrivals {
  int key0 = -1, key1 = -1, key2 = -1, key3 = -1;   // counter indices, -1 when the slot is empty
  int old0 = 0, old1 = 0, old2 = 0, old3 = 0;       // lane 0: value before the add
  int n = 0;
  __device__ __forceinline__ void arrive(int* cnt, int k) {
    __syncwarp();
    const bool l0 = (threadIdx.x & 31) == 0;
    switch (n) {
      case 0: key0 = k; if (l0) old0 = atom_add_acq_rel(cnt + k, 1); break;
      case 1: key1 = k; if (l0) old1 = atom_add_acq_rel(cnt + k, 1); break;
      case 2: key2 = k; if (l0) old2 = atom_add_acq_rel(cnt + k, 1); break;
      default: key3 = k; if (l0) old3 = atom_add_acq_rel(cnt + k, 1); break;
    }
    ++n;
  }
  __device__ __forceinline__ bool full() const { return n >= 4; }
  template <typename F>
  __device__ __forceinline__ void settle(int target, F&& finish) {
    const int keys[4] = {key0, key1, key2, key3};
    const int olds[4] = {old0, old1, old2, old3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i < n) {
        const int o = __shfl_sync(kFull, olds[i], 0);
        __syncwarp();
        if (o == target - 1) finish(keys[i]);
      }
    }
    n = 0;
  }
};

// 2-D tensor copy global -> this CTA's shared memory (one box of `map` at word x, row y), completing
// its bytes on `bar`. x * 4 bytes is a multiple of 16 at every call.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------------------------ grid barrier

// A 64-bit arrival counter in global memory (zeroed at handle creation) that only ever grows: every
// CTA adds 1 at each of the forward's two barriers, so a forward adds 2G. At its start a CTA reads the
// counter; no barrier of this forward can have completed yet (this CTA has not arrived), so the value
// lies in [base, base + G) and base = value - value mod 2G. Barrier b is passed once the counter
// reaches base + b*G. An arrival is one fire-and-forget reduction with release semantics; a wait polls
// with acquire loads and gives up after 1 s (setting the timeout bit and the abort word, which makes
// every later wait of the forward return at once).
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

struct GridBarrier {
  unsigned long long* count;
  int* abort_;
  // One thread per CTA, after the CTA's writes that must be visible are ordered before it by a CTA
  // barrier.
  __device__ __forceinline__ void arrive() const {
    __threadfence();
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(count) : "memory");
  }
  // Bounded wait of one thread until the counter reaches `target`; false on timeout or abort.
  __device__ __forceinline__ bool wait(unsigned long long target, unsigned* err) const {
    if (ld_acquire_u64(count) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (unsigned i = 1;; ++i) {
      __nanosleep(32);
      if (ld_acquire_u64(count) >= target) return true;
      if ((i & 15u) != 0u) continue;               // abort word and clock every 16th poll
      if (ld_relaxed_gpu(abort_) != 0) return false;
      if (globaltimer_ns() - t0 > kWaitNs) {
        atomicOr(err, kErrTimeout);
        atomicExch(abort_, 1);
        return false;
      }
    }
  }
};

// ------------------------------------------------------------------------ 16-bit fixed-point limbs

// m16n8k32 integer MMA, A = int8 weights (16 rows), B = high (signed) or low (unsigned) limb bytes.
__device__ __forceinline__ void imma_hi(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void imma_lo(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stores the warp's 128-segment v (lane l holds the natural elements 4l..4l+3) as 16-bit fixed
// point: q = rint(v / u) with the unit u = 2^(e-14), 2^e <= max|v| < 2^(e+1), so |q| < 2^15;
// q = 256 hi + lo, hi a signed and lo an unsigned byte, in two 128-byte rows. Each 8-element block
// is stored in the order 0,2,4,6,1,3,5,7, the element order of the int8 MMA fragments (the even
// codes of a 32-bit code word, then the odd ones). Lane 0 writes u / 16 (the weights enter the MMA
// as 16c) to *unit.
__device__ __forceinline__ void store_seg_fixed16(uint8_t* hi_row, uint8_t* lo_row, float* unit, const float (&v)[4]) {
  const int lane = threadIdx.x & 31;
  float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  int e = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu) - 127;   // floor(log2 m) for normal m
  e = max(min(e, 100), -100);
  const float up = __uint_as_float(static_cast<uint32_t>(127 + 14 - e) << 23);     // 2^(14-e)
  uint32_t hi = 0, lo = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = min(max(__float2int_rn(v[i] * up), -32768), 32767);
    hi |= static_cast<uint32_t>((q >> 8) & 0xFF) << (8 * i);
    lo |= static_cast<uint32_t>(q & 0xFF) << (8 * i);
  }
  const uint32_t hi_p = __shfl_xor_sync(kFull, hi, 1), lo_p = __shfl_xor_sync(kFull, lo, 1);
  // the even lane of a block pair writes elements 0,2,4,6, the odd lane 1,3,5,7
  const bool odd = lane & 1;
  reinterpret_cast<uint32_t*>(hi_row)[lane] = odd ? __byte_perm(hi_p, hi, 0x7531) : __byte_perm(hi, hi_p, 0x6420);
  reinterpret_cast<uint32_t*>(lo_row)[lane] = odd ? __byte_perm(lo_p, lo, 0x7531) : __byte_perm(lo, lo_p, 0x6420);
  if (lane == 0) *unit = __uint_as_float(static_cast<uint32_t>(127 + e - 18) << 23);    // 2^(e-14) / 16
}

// One 128-wide K group of a 16-row int4 tile (rows g: ra, rows g+8: rb, 16 bytes = 32 codes each)
// against the limbs of token column g (bh, bl: 32 bytes each): exact int32 sums, scaled by f[] into
// the fp32 accumulators (f: {row g, col 2t}, {g, 2t+1}, {g+8, 2t}, {g+8, 2t+1}).
__device__ __forceinline__ void int4_group(float (&acc)[4], const uint4& ra, const uint4& rb, const uint4 (&bh)[2],
                                           const uint4 (&bl)[2], const float (&f)[4]) {
  // two accumulator chains per limb (even and odd steps), so that consecutive MMAs are independent
  int dh[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}}, dl[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
  const uint32_t h[8] = {bh[0].x, bh[0].y, bh[0].z, bh[0].w, bh[1].x, bh[1].y, bh[1].z, bh[1].w};
  const uint32_t l[8] = {bl[0].x, bl[0].y, bl[0].z, bl[0].w, bl[1].x, bl[1].y, bl[1].z, bl[1].w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // even codes of word i (low nibbles) and odd codes (high nibbles), each as the int8 16c
    const uint32_t a0 = (wa[i] << 4) & 0xF0F0F0F0u, a2 = wa[i] & 0xF0F0F0F0u;
    const uint32_t a1 = (wb[i] << 4) & 0xF0F0F0F0u, a3 = wb[i] & 0xF0F0F0F0u;
    imma_hi(dh[i & 1], a0, a1, a2, a3, h[2 * i], h[2 * i + 1]);
    imma_lo(dl[i & 1], a0, a1, a2, a3, l[2 * i], l[2 * i + 1]);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    acc[q] = fmaf(static_cast<float>((dh[0][q] + dh[1][q]) * 256 + dl[0][q] + dl[1][q]), f[q], acc[q]);
}

// One 128-wide K group j of a 16-row NVFP4 tile into two fp32 accumulator sets (steps alternate).
// Codes x E4M3 block scale are exact in fp16; thread t's 32 codes span the blocks 8j+2t and 8j+2t+1,
// whose scales it holds in registers (s0: row g, s1: row g+8; low byte = block 8j+2t).
__device__ __forceinline__ void nvfp4_group_r(float (&acc)[2][4], const uint4& ra, const uint4& rb, const RawB& B,
                                              uint32_t s0, uint32_t s1) {
  uint32_t h0[2], h1[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t a = e4m3_to_half_bits(s0 >> (8 * q)), b = e4m3_to_half_bits(s1 >> (8 * q));
    h0[q] = a | (a << 16);
    h1[q] = b | (b << 16);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w0 = u4_word(ra, i >> 1), w1 = u4_word(rb, i >> 1);
    const int sh = (i & 1) * 16;
    const uint32_t a[4] = {hmul2_u32(e2m1x2_to_half2(w0 >> sh), h0[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w1 >> sh), h1[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w0 >> (sh + 8)), h0[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w1 >> (sh + 8)), h1[i >> 2])};
    mma_f16_16816(acc[i & 1], a, B.b0(i), B.b1(i));
  }
}

// One 128-wide K group of bf16 rows (A) against one or two bf16 operands (B, B2), fp32 accumulation.
__device__ __forceinline__ void bf16_group(float (&acc)[2][4], const RawA<kBf16>& A, const RawB& B, const RawB* B2) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a[4] = {u4_word(A.r0[i >> 1], (2 * i) & 3), u4_word(A.r1[i >> 1], (2 * i) & 3),
                           u4_word(A.r0[i >> 1], (2 * i + 1) & 3), u4_word(A.r1[i >> 1], (2 * i + 1) & 3)};
    mma_bf16_16816(acc[i & 1], a, B.b0(i), B.b1(i));
    if (B2) mma_bf16_16816(acc[(i + 1) & 1], a, B2->b0(i), B2->b1(i));
  }
}

// Rows g < nrows of a bf16 stage (row pitch `pitch`), the other rows of the MMA tile zero.
__device__ __forceinline__ void load_a_bf16_rows(RawA<kBf16>& A, const uint8_t* st, int pitch, int nrows, int g, int jj,
                                                 int t) {
  if (g < nrows) {
    load_a_bf16_smem(A, st + g * pitch, (g + 8 < nrows) ? st + (g + 8) * pitch : nullptr, jj, t);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) A.r0[i] = A.r1[i] = make_uint4(0, 0, 0, 0);
  }
}

// ============================================================================================ route

// Router logits on the tensor cores: rows e0 = c and e1 = c + G of W_r for every token. Routing warp
// rw takes K quarter rw (512 elements = 4 groups); MMA rows 0 and 1 are the two router rows (the
// other 14 rows are zero), columns the tokens (x staged in shared memory). The bf16 products are
// exact and accumulate in fp32 (the router rows are used widened to FP32 on the pages: NInfer
// README, "What is inside"); the four quarters are added in order by routing warp 0.
struct RouterRows {
  uint4 a[4][4];                            // lanes with g < 2: 32 bf16 of row g per group, 4 groups
  __device__ __forceinline__ void load(const DecodeParams& p, int rw, int row) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const bool v = g < 2 && row < p.E;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        a[jj][q] = v ? ld_stream_v4(p.wr + static_cast<size_t>(row) * kH + (4 * rw + jj) * kGroup + 32 * t + 8 * q)
                     : make_uint4(0, 0, 0, 0);
  }
  // partial logits of this warp's quarter into rpart[rw][row 0/1][token]
  __device__ __forceinline__ void mma(const DecodeParams& p, int rw, const uint8_t* xs, int pitch,
                                      float (&rpart)[4][2][kDecodeMaxT]) const {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const bool bv = g < p.T;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      RawA<kBf16> A;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        A.r0[q] = a[jj][q];
        A.r1[q] = make_uint4(0, 0, 0, 0);
      }
      RawB B;
      const uint8_t* q0 = xs + (bv ? g : 0) * pitch + ((4 * rw + jj) * kGroup + 32 * t) * 2;
#pragma unroll
      for (int q = 0; q < 4; ++q) B.u[q] = bv ? *reinterpret_cast<const uint4*>(q0 + 16 * q) : make_uint4(0, 0, 0, 0);
      bf16_group(acc, A, B, nullptr);
    }
    if (g < 2) {
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) rpart[rw][g][2 * t + qq] = acc[0][qq] + acc[1][qq];
    }
  }
};

// One 128-segment of the gate|up activation operand (x in shared memory), written to global memory:
// fp16(Hn x) with every 8-block in the order 0,4,1,5,2,6,3,7 and the 16-bit limbs of Hn x with
// their unit (int4), or fp16(x) (NVFP4).
__device__ void xq_segment(const DecodeParams& p, int tok, int seg, const uint8_t* xs, int pitch) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = *reinterpret_cast<const uint2*>(xs + tok * pitch + (seg * kGroup + 4 * lane) * 2);
  float v[4] = {bf16lo_to_f32(raw.x), bf16hi_to_f32(raw.x), bf16lo_to_f32(raw.y), bf16hi_to_f32(raw.y)};
  if (p.fmt == kInt4) {
    fwht128_warp(v);
    uint8_t* row = p.xq8 + static_cast<size_t>(tok) * (2 * kH) + seg * kGroup;
    store_seg_fixed16(row, row + kH, p.xsc + tok * (kH / kGroup) + seg, v);
  }
  store_seg_half(p.xq + static_cast<size_t>(tok) * kH + seg * kGroup, v, p.fmt == kInt4);
}

// Order-preserving map of a logit to an unsigned key: -0 as +0, NaN as 0 (below every number, so it
// is picked only when nothing else is left); every other key is above 0.
__device__ __forceinline__ unsigned logit_key(float f) {
  unsigned b = __float_as_uint(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_logit(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Routing of a forward in one CTA's shared memory.
struct RouteSmem {
  int ids[kMaxActive];                      // [T][K] selected experts, slots by ascending id
  float w[kMaxActive];                      // [T][K] routing weights
  int inv[kMaxActive];                      // [T][K] permuted position of each (token, slot)
  int cnt[kMaxE];                           // table scratch: counts, then offsets
  unsigned mask[kMaxE];                     // table scratch: token bit masks
  int4 etab[kMaxActive][2];                 // active experts: {e, offset, count, tokens}, {ts_g, ts_u, ts_d, 0}
  int na;                                   // number of active experts
  int wsum[kTabWarps];                      // table scan: per-warp sums
  float rpart[4][2][kDecodeMaxT];           // router: partial logits of the CTA's two rows per K quarter
};

// Logits of one token (one warp): element j of lane l is expert l + 32j (through L2: other CTAs wrote
// them); the keys are formed by make_keys once the loads are back, so that the loads of several
// tokens are in flight together.
__device__ __forceinline__ void load_logits(const DecodeParams& p, int tok, float (&v)[8]) {
  const int lane = threadIdx.x & 31, per = p.E >> 5;
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = (j < per) ? __ldcg(p.logits + tok * p.E + lane + 32 * j) : 0.f;
}
__device__ __forceinline__ void make_keys(const DecodeParams& p, const float (&v)[8], unsigned (&key)[8]) {
  const int per = p.E >> 5;
#pragma unroll
  for (int j = 0; j < 8; ++j) key[j] = (j < per) ? logit_key(v[j]) : 0u;
}

// Top-k of one token (one warp): K rounds of a warp argmax on the fp32 logits. The router is
// unbiased and sigmoid increasing, so the largest logits are the largest scores; ties go to the
// lower id. The slots are listed by ascending expert id and w_k = s_k / max(sum of the chosen s,
// floor), the sum taken in slot order (midagedev/bloomery issue #632, host-policy comment).
__device__ __forceinline__ void topk_select(const DecodeParams& p, int tok, const unsigned (&key)[8], RouteSmem& rs,
                                            bool publish) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, K = p.K, per = E >> 5;
  unsigned taken = 0u;                             // bit j: element j already chosen
  int my_id = 0;
  float my_l = 0.f;
  for (int k = 0; k < K; ++k) {
    // largest key among the elements not yet taken, then the lowest index holding it
    unsigned lm = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per && !((taken >> j) & 1u)) lm = max(lm, key[j]);
    const unsigned gm = __reduce_max_sync(kFull, lm);
    unsigned cand = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 7; j >= 0; --j)
      if (j < per && !((taken >> j) & 1u) && key[j] == gm) cand = static_cast<unsigned>(lane + 32 * j);
    unsigned win = __reduce_min_sync(kFull, cand);
    if (win >= static_cast<unsigned>(E)) win = 0u;   // unreachable: K <= E elements are never all taken
    if ((win & 31u) == static_cast<unsigned>(lane)) taken |= 1u << (win >> 5);
    if (lane == k) { my_id = static_cast<int>(win); my_l = key_logit(gm); }
  }
  int rank = 0;
  for (int k = 0; k < K; ++k) rank += (__shfl_sync(kFull, my_id, k) < my_id);
  const float s = 1.0f / (1.0f + expf(-my_l));
  float s_r = 0.f;                                 // lane r: score of the slot of rank r
  for (int k = 0; k < K; ++k) {
    const float sk = __shfl_sync(kFull, s, k);
    const int rk = __shfl_sync(kFull, rank, k);
    if (rk == lane) s_r = sk;
  }
  float sum = 0.f;
  for (int r = 0; r < K; ++r) sum += __shfl_sync(kFull, s_r, r);
  const float denom = fmaxf(sum, p.floor_);
  if (lane < K) {
    rs.ids[tok * K + rank] = my_id;
    rs.w[tok * K + rank] = s / denom;
    if (publish) {
      p.ids[tok * K + rank] = my_id;
      p.wts[tok * K + rank] = s / denom;
    }
  }
}

// Routing tables from the selected ids, by the CTA's threads (tid; every thread calls it):
// the P = T*K pairs count their experts and set their token bits with shared-memory atomics (sums
// and ORs, so the result does not depend on the order they run in); thread e then holds expert e,
// and one scan over the experts (two 16-bit sums packed in a word: counts and active flags, neither
// above 64) gives every expert its offset and active slot; the active experts' table entries
// {e, offset, count, tokens (4 bits each)}, {ts_g, ts_u, ts_d, 0}; then the expert-major permutation
// (pairs of one expert by ascending token): position p holds t*K+k, inv[t*K+k] = p. With `publish`
// the tables also go to global memory (counts, offsets (E+1), perm, inv, active experts, their
// table) for inspection.
__device__ __forceinline__ void build_tables(const DecodeParams& p, RouteSmem& rs, bool publish, int tid) {
  const int lane = tid & 31, w = tid >> 5;
  const int T = p.T, E = p.E, K = p.K, P = T * K;
  const bool te = tid < kMaxE;                     // threads past the last expert only join the barriers
  if (te) {
    rs.cnt[tid] = 0;
    rs.mask[tid] = 0u;
  }
  __syncthreads();
  if (tid < P) {
    const int id = rs.ids[tid];
    atomicAdd(&rs.cnt[id], 1);
    atomicOr(&rs.mask[id], 1u << (tid / K));
  }
  __syncthreads();
  const int e = tid;
  const int cnt = te && e < E ? rs.cnt[e] : 0;
  const unsigned msk = te ? rs.mask[e] : 0u;
  const unsigned own = static_cast<unsigned>(cnt) | (static_cast<unsigned>(cnt > 0) << 16);
  unsigned inc = own;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const unsigned o = __shfl_up_sync(kFull, inc, m);
    if (lane >= m) inc += o;
  }
  if (lane == 31 && te) rs.wsum[w] = static_cast<int>(inc);
  __syncthreads();
  unsigned before = 0u, total = 0u;
#pragma unroll
  for (int v = 0; v < kTabWarps; ++v) {
    const unsigned x = static_cast<unsigned>(rs.wsum[v]);
    if (v < w) before += x;
    total += x;
  }
  const unsigned ex = before + inc - own;          // exclusive prefix (packed)
  const int off = static_cast<int>(ex & 0xFFFF), slot = static_cast<int>(ex >> 16);
  if (te) rs.cnt[e] = off;                         // every count was read before the barrier above
  if (te && e < E && publish) {
    p.counts[e] = cnt;
    p.offsets[e] = off;
  }
  if (te && e < E && cnt > 0) {
    unsigned toks = 0u, m = msk;
    for (int n = 0; m; ++n) {
      const int tt = __ffs(m) - 1;
      toks |= static_cast<unsigned>(tt) << (4 * n);
      m &= m - 1;
    }
    // weight index: the expert's cache slot when the weights sit in slots, else the expert itself
    const int wi = p.slot_of ? min(max(__ldg(p.slot_of + e), 0), p.n_wslots - 1) : e;
    const float tsg = p.gu_ts ? __ldg(p.gu_ts + 2 * wi) : 1.f;
    const float tsu = p.gu_ts ? __ldg(p.gu_ts + 2 * wi + 1) : 1.f;
    const float tsd = p.dn_ts ? __ldg(p.dn_ts + wi) : 1.f;
    const int4 t0 = make_int4(e, off, cnt, static_cast<int>(toks));
    const int4 t1 = make_int4(__float_as_int(tsg), __float_as_int(tsu), __float_as_int(tsd), wi);
    rs.etab[slot][0] = t0;
    rs.etab[slot][1] = t1;
    if (publish) {
      p.active[slot] = e;
      p.etab[2 * slot] = t0;
      p.etab[2 * slot + 1] = t1;
    }
  }
  if (tid == 0) {
    rs.na = static_cast<int>(total >> 16);
    if (publish) {
      p.offsets[E] = static_cast<int>(total & 0xFFFF);
      *p.n_active = rs.na;
    }
  }
  __syncthreads();
  if (tid < P) {
    const int id = rs.ids[tid], tt = tid / K;
    const int pos = rs.cnt[id] + __popc(rs.mask[id] & ((1u << tt) - 1u));
    rs.inv[tid] = pos;
    if (publish) {
      p.perm[pos] = tid;
      p.inv[tid] = pos;
    }
  }
}

// An expert-table entry; the fields are clamped so that a corrupt table cannot address out of range.
// w is the index of the expert's weights (its cache slot when the weights sit in slots, else e).
struct ExpertInfo {
  int e, w, off, n;
  unsigned toks;
  float tsg, tsu, tsd;
};

// The expert table held by one warp in registers (lane l keeps entries l and l + 32), loaded once;
// an entry is then fetched by shuffles instead of a shared-memory round trip per tile.
struct WarpTable {
  int4 a[2], b[2];
  __device__ __forceinline__ void load(const RouteSmem& rs) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gi = lane + 32 * h;
      a[h] = gi < rs.na ? rs.etab[gi][0] : make_int4(0, 0, 0, 0);
      b[h] = gi < rs.na ? rs.etab[gi][1] : make_int4(0, 0, 0, 0);
    }
  }
  // entry of active slot gi (warp-uniform)
  __device__ __forceinline__ ExpertInfo get(const DecodeParams& p, int gi) const {
    const int h = gi >> 5, src = gi & 31;
    const int4 x = h ? a[1] : a[0], y = h ? b[1] : b[0];
    ExpertInfo r;
    r.e = min(max(__shfl_sync(kFull, x.x, src), 0), p.E - 1);
    r.w = min(max(__shfl_sync(kFull, y.w, src), 0), (p.slot_of ? p.n_wslots : p.E) - 1);
    r.n = min(max(__shfl_sync(kFull, x.z, src), 0), kDecodeMaxT);
    r.off = min(max(__shfl_sync(kFull, x.y, src), 0), p.T * p.K - r.n);
    r.toks = static_cast<unsigned>(__shfl_sync(kFull, x.w, src));
    r.tsg = __int_as_float(__shfl_sync(kFull, y.x, src));
    r.tsu = __int_as_float(__shfl_sync(kFull, y.y, src));
    r.tsd = __int_as_float(__shfl_sync(kFull, y.z, src));
    return r;
  }
};

__device__ __forceinline__ int token_of(const DecodeParams& p, const ExpertInfo& ex, int col) {
  return min(static_cast<int>((ex.toks >> (4 * col)) & 0xFu), p.T - 1);
}

__device__ __forceinline__ int active_count(const DecodeParams& p, const RouteSmem& rs) {
  return min(max(rs.na, 0), min(kMaxActive, p.T * p.K));
}

// ===================================================================================== the kernel

constexpr int kShGuTiles = kIs / 2;         // shared gate|up tiles: 2 hs columns (2 gate + 2 up rows) each
constexpr int kGuTilesPerExpert = kI / 8;   // 64 routed gate|up tiles: 8 h columns (8 gate + 8 up rows) each
constexpr int kTokPitch = 2 * kH + 64;      // bytes per staged token row of x or of the routed operand

// Warps per CTA and the per-warp ring of weight stages. 12 warps (three per scheduler) keep more
// independent MMA chains in flight than 8; the shared memory then holds two stages per warp. int4:
// 4096 B of codes (+256 B for phase C's scales); NVFP4: 4096 B of codes + 512 B of block scales.
template <int FMT>
struct Geom {
  static constexpr int kWarps = 12;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kDepth = 2;
  static constexpr int kStage = FMT == kInt4 ? 4096 + 256 : 4096 + 512;
  static_assert(kWarps >= kRouteWarp0 + kRouteWarps && kWarps * 32 >= kMaxE, "warp roles");
};

template <int FMT>
struct DecShared {
  alignas(128) uint8_t stage[Geom<FMT>::kWarps][Geom<FMT>::kDepth][Geom<FMT>::kStage];
  alignas(16) uint8_t gu_sc[FMT == kInt4 ? Geom<FMT>::kWarps : 1][2][16 * (kH / kGroup) * 2];   // int4: tile scales
  union {
    struct {                                          // phases A and B
      alignas(128) uint8_t xs[kDecodeMaxT][kTokPitch];  // x, bf16
      alignas(128) uint8_t xq[kDecodeMaxT][kTokPitch];  // int4: hi limbs, lo limbs; NVFP4: fp16 x
      float xsc[kDecodeMaxT][kH / kGroup];              // int4: unit / 16 of each segment of xq
    } ab;
    struct {                                          // phase C
      alignas(128) uint8_t hq[kMaxActive][2 * kI];      // down operand of every position: int4 limbs, NVFP4 fp16
      float hsc[kMaxActive][kI / kGroup];               // int4: unit / 16 of each segment of hq
      float opart[kMaxActive][kMaxRowsPerCta];          // routed down outputs of this CTA's rows, per position
      float spart[kShDnSlices][kDecodeMaxT][kMaxRowsPerCta];   // shared down partial sums per K slice
    } c;
  } u;
  RouteSmem rs;
  uint64_t full[Geom<FMT>::kWarps][Geom<FMT>::kDepth];
  uint64_t xbar, xqbar, hqbar, logits_ready;
  unsigned long long bar_base;                        // the grid barriers' counter at the forward's start
};

// A warp's ring position: stages are issued and consumed in one sequence across the three phases.
template <int FMT>
struct Ring {
  static constexpr int D = Geom<FMT>::kDepth;
  uint8_t* base;               // stage[warp][0]
  uint64_t* full;              // full[warp][0]
  int issued = 0, consumed = 0;
  __device__ __forceinline__ uint8_t* slot_ptr(int i) const { return base + (i % D) * Geom<FMT>::kStage; }
  __device__ __forceinline__ uint64_t* bar(int i) const { return full + (i % D); }
  __device__ __forceinline__ bool has_room() const { return issued - consumed < D; }
};

// Bounded wait for a stage (the barrier is the warp's own).
__device__ __forceinline__ void wait_stage(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  if (!mbar_wait_bounded(bar, parity, kWaitNs)) {
    if ((threadIdx.x & 31) == 0) atomicOr(p.err, kErrTimeout);
  }
}

// ---- phase B: gate|up

// Warp-collective: stage q (K groups 4q..4q+3) of gate|up tile `tile` into ring slot i. Shared tile
// st: one tensor box with Sg rows 2st, 2st+1 and one with Su rows 2st, 2st+1 (1 KB each). Routed
// tile (gi, i8): one box of gate rows 8*i8 .. +8 and one of the matching up rows (256 B each); int4
// with q == 0 also the tile's scales (bulk copies into the warp's scale buffer of the tile's
// parity); NVFP4 the block scales of the stage's K quarter (two 8-row boxes of 32 B rows).
template <int FMT>
__device__ void gu_issue(const DecodeParams& p, DecShared<FMT>& sm, Ring<FMT>& ring, int warp, int q, int k, int tile,
                         const ExpertInfo& ex) {
  const int lane = threadIdx.x & 31;
  const int i = ring.issued++;
  uint8_t* st = ring.slot_ptr(i);
  uint64_t* bar = ring.bar(i);
  if (tile < kShGuTiles) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 4 * 1024);
      tma_load_2d(st, &p.tm_sh_gu, q * 256, 2 * tile, bar);
      tma_load_2d(st + 2048, &p.tm_sh_gu, q * 256, kIs + 2 * tile, bar);
    }
    return;
  }
  const int i0 = 8 * ((tile - kShGuTiles) % kGuTilesPerExpert);
  const int erow = ex.w * (2 * kI);
  if constexpr (FMT == kInt4) {
    constexpr uint32_t row_sc = (kH / kGroup) * 2;   // 16 bf16 group scales per row
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 16 * 256 + (q == 0 ? 16 * row_sc : 0));
      tma_load_2d(st, &p.tm_gu, q * 64, erow + i0, bar);
      tma_load_2d(st + 2048, &p.tm_gu, q * 64, erow + kI + i0, bar);
    }
    __syncwarp();
    if (q == 0 && (lane == 1 || lane == 2)) {        // gate rows' scales, then the up rows'
      uint8_t* sc = sm.gu_sc[warp][k & 1] + (lane - 1) * 8 * row_sc;
      bulk_g2s(sc, p.gu_scales + (static_cast<size_t>(erow) + (lane - 1) * kI + i0) * row_sc, 8 * row_sc, bar);
    }
  } else {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 16 * 256 + 16 * 32);
      tma_load_2d(st, &p.tm_gu, q * 64, erow + i0, bar);
      tma_load_2d(st + 2048, &p.tm_gu, q * 64, erow + kI + i0, bar);
      tma_load_2d(st + 4096, &p.tm_gu_sc, q * 8, erow + i0, bar);
      tma_load_2d(st + 4096 + 256, &p.tm_gu_sc, q * 8, erow + kI + i0, bar);
    }
  }
}

// B operand of one group for one thread from a staged token row (32 stored elements, 64 bytes).
__device__ __forceinline__ void load_b_smem(RawB& B, const uint8_t* row, int j, int t, bool valid) {
  if (valid) {
    const uint8_t* q = row + (j * 128 + 32 * t) * 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) B.u[i] = *reinterpret_cast<const uint4*>(q + 16 * i);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) B.u[i] = make_uint4(0, 0, 0, 0);
  }
}

// Limbs (hi row at row, lo row at row + lo_off) of a staged row for group j: the thread's 32 bytes.
__device__ __forceinline__ void load_limbs_smem(uint4 (&bh)[2], uint4 (&bl)[2], const uint8_t* row, int lo_off, int j,
                                                int t, bool valid) {
  if (valid) {
    const uint8_t* ph = row + j * 128 + 32 * t;
    bh[0] = *reinterpret_cast<const uint4*>(ph);
    bh[1] = *reinterpret_cast<const uint4*>(ph + 16);
    bl[0] = *reinterpret_cast<const uint4*>(ph + lo_off);
    bl[1] = *reinterpret_cast<const uint4*>(ph + lo_off + 16);
  } else {
    bh[0] = bh[1] = bl[0] = bl[1] = make_uint4(0, 0, 0, 0);
  }
}

// Last of the 16 tiles of segment seg of an active expert: h -> the down operand (int4: limbs of
// Hn h per 128-segment; NVFP4: fp16 h).
__device__ void finish_segment(const DecodeParams& p, const ExpertInfo& ex, int seg) {
  const int lane = threadIdx.x & 31;
  for (int s = 0; s < ex.n; ++s) {
    const size_t pos = static_cast<size_t>(ex.off + s);
    const float4 hv = __ldcg(reinterpret_cast<const float4*>(p.h32 + pos * kI + seg * kGroup) + lane);
    float v[4] = {hv.x, hv.y, hv.z, hv.w};
    if (p.fmt == kInt4) {
      fwht128_warp(v);
      uint8_t* row = p.hq8 + pos * (2 * kI) + seg * kGroup;
      store_seg_fixed16(row, row + kI, p.hsc + pos * (kI / kGroup) + seg, v);
    } else {
      store_seg_half(p.hq + pos * kI + seg * kGroup, v, false);
    }
  }
}

// ---- phase C: down

// This CTA's rows of y: [r0, r0 + nr).
__device__ __forceinline__ void cta_rows(int& r0, int& nr) {
  const int G = gridDim.x, c = blockIdx.x;
  r0 = (c * kH) / G;
  nr = ((c + 1) * kH) / G - r0;
}

// Warp-collective: phase C item `item` of this CTA into ring slot i. Items 0..7 are the shared
// expert's down rows [r0, r0+16) over K slice 128*item (one 64-word x 16-row tensor box; rows past
// r0+nr belong to the next CTA and are ignored, rows past H read as zero); item 8+gi is active
// expert gi's down rows [r0, r0+nr) over all of K (nr * 256 contiguous bytes of codes) and their
// scales (int4: from the even row at or below r0, an even row count, so that the copy is 16-byte
// aligned; NVFP4: nr rows of 32 B).
template <int FMT>
__device__ void dn_issue(const DecodeParams& p, Ring<FMT>& ring, int item, int r0, int nr, const WarpTable& tab) {
  const int lane = threadIdx.x & 31;
  const int i = ring.issued++;
  uint8_t* st = ring.slot_ptr(i);
  uint64_t* bar = ring.bar(i);
  if (item < kShDnSlices) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 16 * 256);
      tma_load_2d(st, &p.tm_sh_dn, item * 64, r0, bar);
    }
    return;
  }
  const ExpertInfo ex = tab.get(p, item - kShDnSlices);
  const size_t row0 = static_cast<size_t>(ex.w) * kH + r0;
  if (lane == 0) {
    if constexpr (FMT == kInt4) {
      const size_t re = row0 & ~static_cast<size_t>(1);
      const uint32_t nsc = static_cast<uint32_t>(((row0 + nr + 1) & ~static_cast<size_t>(1)) - re);   // even
      mbar_arrive_expect_tx(bar, nr * 256 + nsc * 8);
      bulk_g2s(st, p.dn_codes + row0 * (kI / 2), nr * 256, bar);
      bulk_g2s(st + 4096, p.dn_scales + re * 8, nsc * 8, bar);
    } else {
      mbar_arrive_expect_tx(bar, nr * 256 + nr * 32);
      bulk_g2s(st, p.dn_codes + row0 * (kI / 2), nr * 256, bar);
      bulk_g2s(st + 4096, p.dn_scales + row0 * 32, nr * 32, bar);
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(Geom<FMT>::kThreads, 1) decode_layer_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int D = Geom<FMT>::kDepth;
  constexpr int kWarps = Geom<FMT>::kWarps, kThreads = Geom<FMT>::kThreads;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecShared<FMT>& sm = *reinterpret_cast<DecShared<FMT>*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int G = gridDim.x, c = blockIdx.x;
  const GridBarrier gb{reinterpret_cast<unsigned long long*>(p.cnt + kCntBar), p.cnt + kCntBar + 2};
  Ring<FMT> ring;
  ring.base = &sm.stage[warp][0][0];
  ring.full = &sm.full[warp][0];
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < D; ++i) mbar_init(&sm.full[warp][i], 1);
  }
  if (threadIdx.x == 0) {
    mbar_init(&sm.xbar, 1);
    mbar_init(&sm.xqbar, 1);
    mbar_init(&sm.hqbar, 1);
    mbar_init(&sm.logits_ready, 1);
    const unsigned long long c0 = ld_acquire_u64(gb.count);
    sm.bar_base = c0 - c0 % (2ull * G);
  }
  fence_mbar_init();
  __syncthreads();
  const unsigned long long bar_base = sm.bar_base;

  // ---------------------------------------------------------------- phase A
  // gate|up tile k of this warp (round robin over the CTAs first, then the warps)
  auto tile_of = [&](int k) { return c + G * (warp + kWarps * k); };
  if (threadIdx.x == 0) {                          // x (T token rows), one bulk copy per row
    mbar_arrive_expect_tx(&sm.xbar, p.T * kH * 2);
    for (int r = 0; r < p.T; ++r) bulk_g2s(sm.u.ab.xs[r], p.x + static_cast<size_t>(r) * kH, kH * 2, &sm.xbar);
  }
  int k_issue = 0;                                 // next gate|up stage to issue: tile k_issue >> 2, quarter & 3
  if (warp >= kRouteWarp0 && warp < kRouteWarp0 + kRouteWarps) {
    // router rows c and c + G on the tensor cores (K quarter rw each), then the operand segments
    const int rw = warp - kRouteWarp0, ri = threadIdx.x - kRouteWarp0 * 32;
    RouterRows rr;
    if (!p.route_in) rr.load(p, rw, c + G * g);
    wait_stage(p, &sm.xbar, 0);
    if (!p.route_in) rr.mma(p, rw, sm.u.ab.xs[0], kTokPitch, sm.rs.rpart);
    if (rw == kRouteWarps - 1)
      for (int sg = c; sg < p.T * (kH / kGroup); sg += G)
        xq_segment(p, sg / (kH / kGroup), sg % (kH / kGroup), sm.u.ab.xs[0], kTokPitch);
    named_bar_sync(kBarRoute, kRouteThreads);
    if (rw == 0 && !p.route_in) {                  // quarters added in order: one logit per lane
      const int r = lane >> 3, tok = lane & 7, e = c + G * r;
      if (tok < p.T && e < p.E) {
        const float* q = &sm.rs.rpart[0][r][tok];
        const float v = ((q[0] + q[2 * kDecodeMaxT]) + q[4 * kDecodeMaxT]) + q[6 * kDecodeMaxT];
        __stcg(p.logits + tok * p.E + e, v);
      }
    }
    // ------------------------------------------------------------ barrier 1: logits and operand
    named_bar_sync(kBarRoute, kRouteThreads);
    if (ri == 0) {
      gb.arrive();
      gb.wait(bar_base + G, p.err);
      fence_proxy_async_global();                  // the operand copy below reads other CTAs' writes
      constexpr int kRow = 2 * kH;                 // int4: hi + lo limbs; NVFP4: fp16
      const uint8_t* src = FMT == kInt4 ? p.xq8 : reinterpret_cast<const uint8_t*>(p.xq);
      mbar_arrive_expect_tx(&sm.xqbar, p.T * kRow + (FMT == kInt4 ? p.T * (kH / kGroup) * 4 : 0));
      for (int r = 0; r < p.T; ++r) bulk_g2s(sm.u.ab.xq[r], src + static_cast<size_t>(r) * kRow, kRow, &sm.xqbar);
      if (FMT == kInt4) bulk_g2s(&sm.u.ab.xsc[0][0], p.xsc, p.T * (kH / kGroup) * 4, &sm.xqbar);
      mbar_arrive(&sm.logits_ready);
    }
  } else {
    // the shared expert needs no routing (its tiles fall to warps 0-3; warps 8-11 have no phase A
    // work), but x and the router rows go first: its first gate|up stages (as many as the ring
    // holds) and the L2 fetch of its down rows start once x has landed
    wait_stage(p, &sm.xbar, 0);
    while (ring.has_room() && tile_of(k_issue >> 2) < kShGuTiles) {
      gu_issue<FMT>(p, sm, ring, warp, k_issue & 3, k_issue >> 2, tile_of(k_issue >> 2), ExpertInfo{});
      ++k_issue;
    }
    if (threadIdx.x == 32)
      for (int ch = c; ch < kH * kIs * 2 / 32768; ch += G) prefetch_l2(p.sh_dn + static_cast<size_t>(ch) * 32768, 32768);
  }
  // ---------------------------------------------------------------- phase B: routing (every warp)
  wait_stage(p, &sm.logits_ready, 0);              // barrier 1 is passed: every CTA's logits and operand are in
  if (p.route_in) {                                // the routing is given: ids by ascending id per token
    for (int q = threadIdx.x; q < p.T * p.K; q += kThreads) {
      sm.rs.ids[q] = min(max(__ldcg(p.ids + q), 0), p.E - 1);
      sm.rs.w[q] = __ldcg(p.wts + q);
    }
  } else if (warp < p.T) {                         // token `warp`
    float lv[8];
    unsigned kv[8];
    load_logits(p, warp, lv);
    make_keys(p, lv, kv);
    topk_select(p, warp, kv, sm.rs, c == 0);
  }
  __syncthreads();
  build_tables(p, sm.rs, c == 0, threadIdx.x);
  __syncthreads();
  const int na = active_count(p, sm.rs);
  WarpTable tab;
  tab.load(sm.rs);
  auto info = [&](int tl) {
    ExpertInfo ex{};
    if (tl >= kShGuTiles) ex = tab.get(p, (tl - kShGuTiles) / kGuTilesPerExpert);
    return ex;
  };
  const int n_gu = kShGuTiles + kGuTilesPerExpert * na;   // gate|up tiles of the forward
  int r0, nr;
  cta_rows(r0, nr);
  const int n_items = kShDnSlices + na;            // phase C items of this CTA
  // ---------------------------------------------------------------- phase B: gate|up tiles
  bool have_xq = false;
  PendingArrivals seg_arr;
  auto finish_last = [&](int key) {            // this warp completed the segment: rotate it
    const int gi = (key - kCntSeg) / 4, seg = (key - kCntSeg) % 4;
    finish_segment(p, tab.get(p, gi), seg);
    if (lane == 0) p.cnt[key] = 0;
  };
  float acc[2][4];
  ExpertInfo ex{};
  bool bvalid = false;
  int tok0 = 0, tok1 = 0;                          // tokens of MMA columns 2t, 2t+1
  const uint8_t* brow = nullptr;                   // this lane's activation row (column g)
  auto refill = [&]() {                            // keep the ring full
    while (ring.has_room() && tile_of(k_issue >> 2) < n_gu) {
      const int tk = tile_of(k_issue >> 2);
      gu_issue<FMT>(p, sm, ring, warp, k_issue & 3, k_issue >> 2, tk, info(tk));
      ++k_issue;
    }
  };
  for (int s = 0;; ++s) {
    const int k = s >> 2, q = s & 3, tl = tile_of(k);
    if (q == 0 && tl >= n_gu) break;
    refill();
    if (q == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[0][i] = acc[1][i] = 0.f;
      if (tl >= kShGuTiles) {
        if (!have_xq) {
          wait_stage(p, &sm.xqbar, 0);
          have_xq = true;
        }
        ex = info(tl);
        bvalid = g < ex.n;
        tok0 = token_of(p, ex, 2 * t);
        tok1 = token_of(p, ex, 2 * t + 1);
        brow = sm.u.ab.xq[bvalid ? token_of(p, ex, g) : 0];
      }
    }
    const int i = ring.consumed;
    wait_stage(p, ring.bar(i), (i / D) & 1);
    const uint8_t* st = ring.slot_ptr(i);
    if (tl < kShGuTiles) {
      // rows g = 0,1: gate 2tl, 2tl+1; g = 2,3: up 2tl, 2tl+1; MMA rows 4..15 are zero
      const bool xv = g < p.T;
      const uint8_t* xr = sm.u.ab.xs[xv ? g : 0];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        RawA<kBf16> A;
        load_a_bf16_rows(A, st, 1024, 4, g, jj, t);
        RawB B;
        load_b_smem(B, xr, 4 * q + jj, t, xv);
        bf16_group(acc, A, B, nullptr);
      }
    } else {
      // routed: the stage's codes (and NVFP4 block scales: gate rows 8 x 32 B at 4096, up rows at
      // 4352, blocks of this K quarter) go to registers, and the slot is refilled before the MMAs
      uint4 ra[4], rb[4];
      uint32_t bs0[4], bs1[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        ra[jj] = *reinterpret_cast<const uint4*>(st + g * 256 + jj * 64 + 16 * t);
        rb[jj] = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + jj * 64 + 16 * t);
        if constexpr (FMT != kInt4) {
          bs0[jj] = *reinterpret_cast<const uint16_t*>(st + 4096 + g * 32 + jj * 8 + 2 * t);
          bs1[jj] = *reinterpret_cast<const uint16_t*>(st + 4096 + 256 + g * 32 + jj * 8 + 2 * t);
        }
      }
      __syncwarp();                                // every lane's reads of the slot precede its refill
      ring.consumed++;
      refill();
      if constexpr (FMT == kInt4) {
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(sm.gu_sc[warp][k & 1]);
        const bool v0 = 2 * t < ex.n, v1 = 2 * t + 1 < ex.n;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = 4 * q + jj;
          uint4 bh[2], bl[2];
          load_limbs_smem(bh, bl, brow, kH, j, t, bvalid);
          const float sg = bf16_bits_to_f32(sc[g * 16 + j]), su = bf16_bits_to_f32(sc[(8 + g) * 16 + j]);
          const float x0 = v0 ? sm.u.ab.xsc[tok0][j] : 0.f, x1 = v1 ? sm.u.ab.xsc[tok1][j] : 0.f;
          const float f[4] = {sg * x0, sg * x1, su * x0, su * x1};
          int4_group(acc[0], ra[jj], rb[jj], bh, bl, f);
        }
      } else {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          RawB B;
          load_b_smem(B, brow, 4 * q + jj, t, bvalid);
          nvfp4_group_r(acc, ra[jj], rb[jj], B, bs0[jj], bs1[jj]);
        }
      }
    }
    if (tl < kShGuTiles) {
      __syncwarp();                                // every lane's reads of the slot precede its refill
      ring.consumed++;
    }
    if (q != 3) continue;
    // ---- tile epilogue
    float cc[4];
#pragma unroll
    for (int i2 = 0; i2 < 4; ++i2) cc[i2] = acc[0][i2] + acc[1][i2];
    if (tl < kShGuTiles) {
      const float u0 = __shfl_down_sync(kFull, cc[0], 8), u1 = __shfl_down_sync(kFull, cc[1], 8);
      if (g < 2) {
        const float uv[2] = {u0, u1};
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int tok = 2 * t + qq;
          if (tok < p.T) {
            const float hs = silu(cc[qq]) * uv[qq];
            const uint16_t hi = f32_to_bf16_bits(hs);
            const uint16_t lo = f32_to_bf16_bits(hs - bf16_bits_to_f32(hi));
            p.hs_hi[tok * kIs + 2 * tl + g] = hi;
            p.hs_lo[tok * kIs + 2 * tl + g] = lo;
          }
        }
      }
    } else {
      const int r = tl - kShGuTiles, gi = r / kGuTilesPerExpert, i8 = r % kGuTilesPerExpert;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int col = 2 * t + qq;
        if (col < ex.n)
          p.h32[static_cast<size_t>(ex.off + col) * kI + 8 * i8 + g] = silu(cc[qq] * ex.tsg) * (cc[2 + qq] * ex.tsu);
      }
      const int seg = i8 / (kGroup / 8);
      if (seg_arr.full()) seg_arr.settle(kGroup / 8, finish_last);
      seg_arr.arrive(p.cnt, kCntSeg + 4 * gi + seg);
    }
  }
  seg_arr.settle(kGroup / 8, finish_last);
  if (warp == kRouteWarp0 && !have_xq) wait_stage(p, &sm.xqbar, 0);   // no copy may still write the operand rows

  // ---------------------------------------------------------------- phase C: first stages, barrier 2
  int it_issue = warp;                             // this warp's items: warp, warp + 8, ...
  while (ring.has_room() && it_issue < n_items) {
    dn_issue<FMT>(p, ring, it_issue, r0, nr, tab);
    it_issue += kWarps;
  }
  __syncthreads();                                 // every warp's h, hs and operand writes are done
  if (threadIdx.x == 0) {
    gb.arrive();
    gb.wait(bar_base + 2ull * G, p.err);
    fence_proxy_async_global();
    const int P = p.T * p.K;
    const uint8_t* src = FMT == kInt4 ? p.hq8 : reinterpret_cast<const uint8_t*>(p.hq);
    mbar_arrive_expect_tx(&sm.hqbar, P * 2 * kI + (FMT == kInt4 ? P * (kI / kGroup) * 4 : 0));
    bulk_g2s(&sm.u.c.hq[0][0], src, P * 2 * kI, &sm.hqbar);
    if (FMT == kInt4) bulk_g2s(&sm.u.c.hsc[0][0], p.hsc, P * (kI / kGroup) * 4, &sm.hqbar);
  }
  __syncthreads();                                 // the grid barrier is passed for every thread

  // ---------------------------------------------------------------- phase C: down items
  bool have_hq = false;
  auto release = [&]() {                           // the slot is read: refill it with the next item
    __syncwarp();
    ring.consumed++;
    if (it_issue < n_items) {
      dn_issue<FMT>(p, ring, it_issue, r0, nr, tab);
      it_issue += kWarps;
    }
  };
  for (int it = warp; it < n_items; it += kWarps) {
    const int i = ring.consumed;
    wait_stage(p, ring.bar(i), (i / D) & 1);
    const uint8_t* st = ring.slot_ptr(i);
    float dacc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) dacc[a][b] = 0.f;
    if (it < kShDnSlices) {
      // rows g, g+8 of the box (row r at r * 256: K elements 128j .. 128j + 127, bf16) against K
      // slice j of hs (bf16 hi + lo pair, written by other CTAs: read through L2)
      const int j = it;
      const bool bv = g < p.T;
      const size_t r = static_cast<size_t>(bv ? g : 0) * kIs;
      RawB Bh, Bl;
      Bh.load_cg(p.hs_hi + r, j, t, bv);
      Bl.load_cg(p.hs_lo + r, j, t, bv);
      RawA<kBf16> A;
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        A.r0[qd] = *reinterpret_cast<const uint4*>(st + g * 256 + (32 * t) * 2 + 16 * qd);
        A.r1[qd] = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + (32 * t) * 2 + 16 * qd);
      }
      release();
      bf16_group(dacc, A, Bh, &Bl);
      float cs[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) cs[b] = dacc[0][b] + dacc[1][b];
      // {row g, tok 2t}, {g, 2t+1}, {g+8, 2t}, {g+8, 2t+1}
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int tok = 2 * t + (b & 1), row = g + 8 * (b >> 1);
        if (tok < p.T) sm.u.c.spart[j][tok][row] = cs[b];
      }
    } else {
      // rows g, g+8 of the stage (row r at r * 256); rows >= nr are the next expert's or beyond:
      // they are read (inside the stage) but their results are dropped. Codes and scales go to
      // registers and the slot is refilled before the MMAs.
      const int ga = min(g, nr - 1), gb2 = min(g + 8, nr - 1);
      uint4 ra[4], rb[4];
      uint32_t sa[4], sb[4];                       // int4: f32 bits of the group scales; NVFP4: 2 E4M3 bytes
#pragma unroll
      for (int j = 0; j < kI / kGroup; ++j) {
        ra[j] = *reinterpret_cast<const uint4*>(st + g * 256 + j * 64 + 16 * t);
        rb[j] = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + j * 64 + 16 * t);
        if constexpr (FMT == kInt4) {
          // row r's 4 bf16 scales at 4096 + (r + (r0 & 1)) * 8 (the copy starts at an even row)
          const uint16_t* s16 = reinterpret_cast<const uint16_t*>(st + 4096) + (r0 & 1) * 4;
          sa[j] = static_cast<uint32_t>(s16[ga * 4 + j]) << 16;
          sb[j] = static_cast<uint32_t>(s16[gb2 * 4 + j]) << 16;
        } else {
          sa[j] = *reinterpret_cast<const uint16_t*>(st + 4096 + ga * 32 + j * 8 + 2 * t);
          sb[j] = *reinterpret_cast<const uint16_t*>(st + 4096 + gb2 * 32 + j * 8 + 2 * t);
        }
      }
      release();
      if (!have_hq) {
        wait_stage(p, &sm.hqbar, 0);
        have_hq = true;
      }
      const ExpertInfo e2 = tab.get(p, it - kShDnSlices);
      const bool bv = g < e2.n;
      const uint8_t* hrow = sm.u.c.hq[e2.off + (bv ? g : 0)];
      if constexpr (FMT == kInt4) {
        const bool v0 = 2 * t < e2.n, v1 = 2 * t + 1 < e2.n;
        const float* x0p = sm.u.c.hsc[e2.off + (v0 ? 2 * t : 0)];
        const float* x1p = sm.u.c.hsc[e2.off + (v1 ? 2 * t + 1 : 0)];
#pragma unroll
        for (int j = 0; j < kI / kGroup; ++j) {
          uint4 bh[2], bl[2];
          load_limbs_smem(bh, bl, hrow, kI, j, t, bv);
          const float s0 = __uint_as_float(sa[j]), s1 = __uint_as_float(sb[j]);
          const float x0 = v0 ? x0p[j] : 0.f, x1 = v1 ? x1p[j] : 0.f;
          const float f[4] = {s0 * x0, s0 * x1, s1 * x0, s1 * x1};
          int4_group(dacc[0], ra[j], rb[j], bh, bl, f);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kI / kGroup; ++j) {
          RawB B;
          load_b_smem(B, hrow, j, t, bv);
          nvfp4_group_r(dacc, ra[j], rb[j], B, sa[j], sb[j]);
        }
      }
      float cs[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) cs[b] = dacc[0][b] + dacc[1][b];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int col = 2 * t + (b & 1), row = g + 8 * (b >> 1);
        if (col < e2.n) sm.u.c.opart[e2.off + col][row] = cs[b] * e2.tsd;
      }
    }
  }
  if (warp == 0 && !have_hq) wait_stage(p, &sm.hqbar, 0);   // no copy may still write this CTA's memory
  __syncthreads();
  // ---------------------------------------------------------------- combine this CTA's rows
  for (int idx = threadIdx.x; idx < p.T * nr; idx += kThreads) {
    const int tok = idx / nr, rl = idx % nr, n = r0 + rl;
    float ys = 0.f;
#pragma unroll
    for (int j = 0; j < kShDnSlices; ++j) ys += sm.u.c.spart[j][tok][rl];
    float a = 0.f;
    for (int k = 0; k < p.K; ++k) {
      const int q = tok * p.K + k;
      const int pos = min(max(sm.rs.inv[q], 0), p.T * p.K - 1);
      a = fmaf(sm.rs.w[q], sm.u.c.opart[pos][rl], a);
    }
    p.ys[tok * kH + n] = ys;
    p.y[tok * kH + n] = f32_to_bf16_bits(fmaf(p.routed_scale, a, ys));
  }
}

// Dynamic shared memory limit and the carve-out, once per kernel.
template <typename Kern>
cudaError_t allow_smem(Kern kernel, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

}  // namespace

size_t decode_smem_bytes(int fmt) { return fmt == kInt4 ? sizeof(DecShared<kInt4>) : sizeof(DecShared<kNvfp4>); }

cudaError_t decode_check_residency(int fmt, int* blocks_per_sm) {
  const size_t smem = decode_smem_bytes(fmt);
  cudaError_t e = fmt == kInt4 ? allow_smem(decode_layer_kernel<kInt4>, smem)
                               : allow_smem(decode_layer_kernel<kNvfp4>, smem);
  if (e != cudaSuccess) return e;
  return fmt == kInt4
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, decode_layer_kernel<kInt4>,
                                                             Geom<kInt4>::kThreads, smem)
             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, decode_layer_kernel<kNvfp4>,
                                                             Geom<kNvfp4>::kThreads, smem);
}

cudaError_t launch_decode(const DecodeParams& p, int n_sm, cudaStream_t s) {
  static_assert(sizeof(DecShared<kInt4>) <= 227 * 1024 && sizeof(DecShared<kNvfp4>) <= 227 * 1024,
                "shared memory per CTA");
  const size_t smem = decode_smem_bytes(p.fmt);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(p.fmt == kInt4 ? Geom<kInt4>::kThreads : Geom<kNvfp4>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;     // every CTA resident at once: the grid barriers need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return p.fmt == kInt4 ? cudaLaunchKernelEx(&cfg, decode_layer_kernel<kInt4>, p)
                        : cudaLaunchKernelEx(&cfg, decode_layer_kernel<kNvfp4>, p);
}

}  // namespace flint
