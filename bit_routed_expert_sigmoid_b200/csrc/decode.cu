// Whole-layer forward for small token counts (T <= 8): three kernels chained by programmatic
// dependent launch (PDL), none of which ever waits for another CTA.
//
// A decode forward streams 23-92 MB of weights through the chain router -> selection -> gate|up ->
// down -> combine. Each arrow of that chain is a kernel boundary here, and PDL hides it: the next
// kernel is resident and streaming weights that do not depend on the previous one before that one
// has finished, and it calls griddepcontrol.wait only before it reads what the previous one wrote.
//
//   route    CTAs split the router rows (fp32 logits) and the activation operand of gate|up; the
//            last CTA to finish (atomic arrival counter) selects the top-k of every token and builds
//            the routing tables. It lets the gate|up kernel launch at once.
//   gate_up  persistent, one CTA per SM; every warp runs its own pipeline: its lanes bring 4 KB
//            stages of weight rows from HBM into the warp's shared-memory ring with bulk copies
//            (cp.async.bulk + mbarrier transaction counts) and the warp turns them into tensor-core
//            products with the activations. Shared-expert tiles come first and need no routing, so
//            they stream while the route kernel still runs; the routed tiles follow after
//            griddepcontrol.wait. The warp that finishes the last of the 16 tiles of a 128-segment
//            of h turns that segment into the down operand.
//   down     same pipelines; the first weight stages are requested before griddepcontrol.wait, so
//            HBM stays busy through the tail of gate_up. The warp that finishes the last tile of a
//            64-row block of y combines that block: y = bf16(routed_scale * sum_k w_k o_k + ys).
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
// Every wait is either the hardware grid dependency or an mbarrier wait on the warp's own copies;
// the latter is bounded and records a timeout bit in the error word when it expires.
#include "frag.cuh"
#include "kernels.cuh"

namespace flint {

namespace {

#ifndef FLINT_WAIT_NS
#define FLINT_WAIT_NS 1000000000ull          // 1 s
#endif
constexpr uint64_t kWaitNs = FLINT_WAIT_NS;
constexpr unsigned kFull = 0xFFFFFFFFu;

// Asks L2 to fetch [ptr, ptr + bytes) from HBM (a hint; no completion to wait for).
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Arrival of the calling thread on a counter with acquire-release semantics at GPU scope; returns
// the previous value.
__device__ __forceinline__ int atom_add_acq_rel(int* ctr, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(ctr), "r"(v) : "memory");
  return old;
}

// A warp's arrival on a counter whose result is examined later: the warp barrier orders every
// lane's earlier global writes before lane 0's release; the returned value is only waited for when
// settle() reads it (typically one tile later), so the atomic's latency overlaps the next tile.
// settle() returns the counter index if this arrival brought the counter to `target` (the warp is
// the last arriver, and lane 0's acquire precedes every lane's later reads), else -1.
struct PendingArrival {
  int key = -1;                             // counter index, -1 when nothing is pending
  int target = 0;
  int old = 0;                              // lane 0: value before the add
  __device__ __forceinline__ void arrive(int* cnt, int k, int tgt) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) old = atom_add_acq_rel(cnt + k, 1);
    key = k;
    target = tgt;
  }
  __device__ __forceinline__ int settle() {
    if (key < 0) return -1;
    const int o = __shfl_sync(kFull, old, 0);
    const int k = key;
    key = -1;
    __syncwarp();
    return o == target - 1 ? k : -1;
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

// One 128-wide K group of a 16-row NVFP4 tile into two fp32 accumulator sets (steps alternate).
// Codes x E4M3 block scale are exact in fp16; thread t's 32 codes span the blocks 8j+2t, 8j+2t+1.
__device__ __forceinline__ void nvfp4_group(float (&acc)[2][4], const uint4& ra, const uint4& rb, const RawB& B,
                                            const uint8_t* bs0, const uint8_t* bs1, int j, int t) {
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
    const uint32_t w0 = u4_word(ra, i >> 1), w1 = u4_word(rb, i >> 1);
    const int sh = (i & 1) * 16;
    const uint32_t a[4] = {hmul2_u32(e2m1x2_to_half2(w0 >> sh), s0[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w1 >> sh), s1[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w0 >> (sh + 8)), s0[i >> 2]),
                           hmul2_u32(e2m1x2_to_half2(w1 >> (sh + 8)), s1[i >> 2])};
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
    load_a_bf16_smem(A, st + g * pitch, nullptr, jj, t);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) A.r0[i] = A.r1[i] = make_uint4(0, 0, 0, 0);
  }
}

// ============================================================================================ route

constexpr int kRouteWarps = 8;

// 8 bf16 x 8 bf16 dot product; the products are exact in fp32.
__device__ __forceinline__ float dot8_bf16(const uint4& a, const uint4& b, float acc) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc = fmaf(bf16lo_to_f32(aw[q]), bf16lo_to_f32(bw[q]), acc);
    acc = fmaf(bf16hi_to_f32(aw[q]), bf16hi_to_f32(bw[q]), acc);
  }
  return acc;
}

__device__ __forceinline__ void load_router_row(uint4 (&w)[8], const DecodeParams& p, int e) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = ld_stream_v4(p.wr + static_cast<size_t>(e) * kH + 8 * lane + 256 * i);
}

// logits[t][e] for every token (one warp, router row in w; lane l covers elements 8l + 256i; x in
// shared memory).
__device__ void route_row(const DecodeParams& p, int e, const uint4 (&w)[8], const uint16_t* xs) {
  const int lane = threadIdx.x & 31;
  float acc[kDecodeMaxT];
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) {
    acc[t] = 0.f;
    if (t < p.T) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        acc[t] = dot8_bf16(w[i], *reinterpret_cast<const uint4*>(xs + t * kH + 8 * lane + 256 * i), acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) acc[t] += __shfl_xor_sync(kFull, acc[t], m);
    if (lane == 0 && t < p.T) p.logits[t * p.E + e] = acc[t];
  }
}

// One 128-segment of the gate|up activation operand (x in shared memory), written to global memory:
// fp16(Hn x) with every 8-block in the order 0,4,1,5,2,6,3,7 and the 16-bit limbs of Hn x with
// their unit (int4), or fp16(x) (NVFP4).
__device__ void xq_segment(const DecodeParams& p, int tok, int seg, const uint16_t* xs) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = *reinterpret_cast<const uint2*>(xs + tok * kH + seg * kGroup + 4 * lane);
  float v[4] = {bf16lo_to_f32(raw.x), bf16hi_to_f32(raw.x), bf16lo_to_f32(raw.y), bf16hi_to_f32(raw.y)};
  if (p.fmt == kInt4) {
    fwht128_warp(v);
    uint8_t* row = p.xq8 + static_cast<size_t>(tok) * (2 * kH) + seg * kGroup;
    store_seg_fixed16(row, row + kH, p.xsc + tok * (kH / kGroup) + seg, v);
  }
  store_seg_half(p.xq + static_cast<size_t>(tok) * kH + seg * kGroup, v, p.fmt == kInt4);
}

// Order-preserving map of a float (not NaN) to an unsigned integer; -0 maps like +0.
__device__ __forceinline__ unsigned float_key(float f) {
  unsigned b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Routing of a forward in one CTA's shared memory. Every projection CTA derives it from the logits
// (top-k and tables are a few microseconds of work for T <= 8): a CTA never waits for another.
struct RouteSmem {
  int ids[kMaxActive];                      // [T][K] selected experts, slots by ascending id
  float w[kMaxActive];                      // [T][K] routing weights
  int inv[kMaxActive];                      // [T][K] permuted position of each (token, slot)
  int cnt[kMaxE];                           // table scratch: counts, then offsets
  unsigned mask[kMaxE];                     // table scratch: token bit masks
  int4 etab[kMaxActive][2];                 // active experts: {e, offset, count, tokens}, {ts_g, ts_u, ts_d, 0}
  int na;                                   // number of active experts
};

// Top-k of one token (one warp): K rounds of a warp argmax on the fp32 logits. The router is
// unbiased and sigmoid increasing, so the largest logits are the largest scores; ties go to the
// lower id. The slots are listed by ascending expert id and w_k = s_k / max(sum of the chosen s,
// floor), the sum taken in slot order (midagedev/bloomery issue #632, host-policy comment).
__device__ __forceinline__ void topk_token(const DecodeParams& p, int tok, RouteSmem& rs, bool publish) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, K = p.K, per = E >> 5;
  const float floor_ = p.floor_;
  const float* logits = p.logits;
  int* g_ids = p.ids;
  float* g_wts = p.wts;
  // element j of lane l is expert l + 32j; key 0 marks an element that is absent or taken (every
  // finite logit has a key above 0)
  unsigned key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) key[j] = (j < per) ? float_key(__ldcg(logits + tok * E + lane + 32 * j)) : 0u;
  int my_id = 0;
  float my_l = 0.f;
  for (int k = 0; k < K; ++k) {
    // largest logit: one warp max-reduction of the keys; then the lowest index holding it
    unsigned lm = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) lm = max(lm, key[j]);
    const unsigned gm = __reduce_max_sync(kFull, lm);
    unsigned cand = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 7; j >= 0; --j)
      if (key[j] == gm) cand = static_cast<unsigned>(lane + 32 * j);
    unsigned win = __reduce_min_sync(kFull, cand);
    if (win >= static_cast<unsigned>(E)) win = 0u;  // unreachable with finite logits
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (win == static_cast<unsigned>(lane + 32 * j)) key[j] = 0u;
    if (lane == k) { my_id = static_cast<int>(win); my_l = key_float(gm); }
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
  const float denom = fmaxf(sum, floor_);
  if (lane < K) {
    rs.ids[tok * K + rank] = my_id;
    rs.w[tok * K + rank] = s / denom;
    if (publish) {
      g_ids[tok * K + rank] = my_id;
      g_wts[tok * K + rank] = s / denom;
    }
  }
}

// Routing tables from the selected ids (one warp): the experts with tokens (ascending) and their
// table, and the expert-major permutation (pairs of one expert by ascending token): position p
// holds t*K+k, inv[t*K+k] = p. Ranks come from bit masks and scans, so the result does not depend
// on the order atomics run in. With `publish` the tables also go to global memory (counts,
// offsets (E+1), perm, inv, active experts, their table) for inspection.
__device__ __forceinline__ void build_tables(const DecodeParams& p, RouteSmem& rs, bool publish) {
  int* scr_cnt = rs.cnt;
  unsigned* scr_mask = rs.mask;
  const int* s_ids = rs.ids;
  const int lane = threadIdx.x & 31;
  const int T = p.T, E = p.E, K = p.K, P = T * K;
  // parameters in registers: the table stores below could otherwise force them to be reloaded
  const float* gu_ts = p.gu_ts;
  const float* dn_ts = p.dn_ts;
  int* g_counts = p.counts;
  int* g_offsets = p.offsets;
  int* g_active = p.active;
  int4* g_etab = p.etab;
  int* g_n_active = p.n_active;
  int* g_perm = p.perm;
  int* g_inv = p.inv;
  for (int e = lane; e < kMaxE; e += 32) {
    scr_cnt[e] = 0;
    scr_mask[e] = 0u;
  }
  __syncwarp();
  const int id0 = lane < P ? s_ids[lane] : 0, id1 = lane + 32 < P ? s_ids[lane + 32] : 0;
  if (lane < P) { atomicAdd(&scr_cnt[id0], 1); atomicOr(&scr_mask[id0], 1u << (lane / K)); }
  if (lane + 32 < P) { atomicAdd(&scr_cnt[id1], 1); atomicOr(&scr_mask[id1], 1u << ((lane + 32) / K)); }
  __syncwarp();
  // lane holds experts 8*lane .. 8*lane+7 (loops kept rolled: this code runs once per CTA, where
  // instruction fetches dominate)
  int s = 0, a = 0;
#pragma unroll 1
  for (int j = 0; j < 8; ++j) {
    const int e = 8 * lane + j;
    const int c = e < E ? scr_cnt[e] : 0;
    s += c;
    a += c > 0;
  }
  int si = s, ai = a;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int os = __shfl_up_sync(kFull, si, m), oa = __shfl_up_sync(kFull, ai, m);
    if (lane >= m) { si += os; ai += oa; }
  }
  int off = si - s, slot = ai - a;
  __syncwarp();
#pragma unroll 1
  for (int j = 0; j < 8; ++j) {
    const int e = 8 * lane + j;
    if (e >= E) break;
    const int c = scr_cnt[e];
    if (publish) {
      g_counts[e] = c;
      g_offsets[e] = off;
    }
    scr_cnt[e] = off;
    if (c > 0) {
      const unsigned m = scr_mask[e];
      unsigned toks = 0;
      int n = 0;
#pragma unroll 1
      for (int tt = 0; tt < T; ++tt)
        if ((m >> tt) & 1u) toks |= static_cast<unsigned>(tt) << (4 * n++);
      const float tsg = gu_ts ? __ldg(gu_ts + 2 * e) : 1.f;
      const float tsu = gu_ts ? __ldg(gu_ts + 2 * e + 1) : 1.f;
      const float tsd = dn_ts ? __ldg(dn_ts + e) : 1.f;
      const int4 t0 = make_int4(e, off, c, static_cast<int>(toks));
      const int4 t1 = make_int4(__float_as_int(tsg), __float_as_int(tsu), __float_as_int(tsd), 0);
      rs.etab[slot][0] = t0;
      rs.etab[slot][1] = t1;
      if (publish) {
        g_active[slot] = e;
        g_etab[2 * slot] = t0;
        g_etab[2 * slot + 1] = t1;
      }
      ++slot;
    }
    off += c;
  }
  if (lane == 31) {
    rs.na = ai;
    if (publish) {
      g_offsets[E] = si;
      *g_n_active = ai;
    }
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = lane + 32 * h;
    if (q < P) {
      const int id = h ? id1 : id0, tt = q / K;
      const int pos = scr_cnt[id] + __popc(scr_mask[id] & ((1u << tt) - 1u));
      rs.inv[q] = pos;
      if (publish) {
        g_perm[pos] = q;
        g_inv[q] = pos;
      }
    }
  }
}

// A group of `nw` warps (group-relative warp index gw; named barrier `bar` over the group's
// threads): top-k of every token (a token per warp), then the tables (the group's first warp).
__device__ __noinline__ void route_group(const DecodeParams& p, RouteSmem& rs, bool publish, int gw, int nw,
                                            int bar) {
  for (int tok = gw; tok < p.T; tok += nw) topk_token(p, tok, rs, publish);
  named_bar_sync(bar, nw * 32);
  if (gw == 0) build_tables(p, rs, publish);
  named_bar_sync(bar, nw * 32);
}

__global__ void __launch_bounds__(kRouteWarps * 32) decode_route_kernel(const __grid_constant__ DecodeParams p) {
  pdl_trigger();                                   // the gate|up kernel may start its shared-expert tiles
  __shared__ __align__(128) uint16_t xs[kDecodeMaxT * kH];
  __shared__ uint64_t xbar;
  const int warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * kRouteWarps + warp, nw = gridDim.x * kRouteWarps;
  if (threadIdx.x == 0) {                          // x (T contiguous rows) by one bulk copy
    mbar_init(&xbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&xbar, p.T * kH * 2);
    bulk_g2s(xs, p.x, p.T * kH * 2, &xbar);
  }
  uint4 w[8];
  if (gw < p.E) load_router_row(w, p, gw);
  __syncthreads();                                 // the barrier is initialised
  if (!mbar_wait_bounded(&xbar, 0, kWaitNs) && threadIdx.x == 0) atomicOr(p.err, kErrTimeout);
  for (int e = gw; e < p.E; e += nw) {
    if (e != gw) load_router_row(w, p, e);
    route_row(p, e, w, xs);
  }
  for (int sg = gw; sg < p.T * (kH / kGroup); sg += nw) xq_segment(p, sg / (kH / kGroup), sg % (kH / kGroup), xs);
}

// ================================================================================ weight pipelines

constexpr int kShGuTiles = kIs / 2;         // shared gate|up tiles: 2 hs columns each
constexpr int kShDnTiles = kH / 8;          // shared down tiles: 8 ys rows each, in 4 stages
constexpr int kGuTilesPerExpert = kI / 8;   // 64 routed gate|up tiles: 8 h columns each
constexpr int kDnTilesPerExpert = kH / 32;  // 64 routed down tiles: 32 o rows each


constexpr int kDnStage = 4096 + 512;        // codes (16 rows x 256 B, or 8 bf16 rows x 512 B) + scales
// int4 runs 16 warps with 2-stage rings (at most 128 registers), NVFP4 8 warps with 4 stages; about
// 128 KB per SM in flight, and the rest of the SM's 256 KB holds L1 lines of the activation rows.
template <int FMT>
struct DnGeom {
  static constexpr int kWarps = FMT == kInt4 ? 16 : 8;
  static constexpr int kDepth = FMT == kInt4 ? 2 : 4;
};
template <int FMT>
struct DnWarp {
  alignas(128) uint8_t stage[DnGeom<FMT>::kDepth][kDnStage];
  uint64_t full[DnGeom<FMT>::kDepth];
};
template <int FMT>
struct DnShared {
  DnWarp<FMT> w[DnGeom<FMT>::kWarps];
  RouteSmem rs;
  alignas(128) uint8_t hq[kMaxActive][2 * kI];        // down operand of every position: int4 limbs (hi, lo), NVFP4 fp16
  float hsc[kMaxActive][kI / kGroup];                 // int4: unit / 16 of each segment of hq
  uint64_t hqbar;                                     // completion of the operand copy
};

// Bounded wait for a stage (the barrier is the warp's own).
__device__ __forceinline__ void wait_stage(const DecodeParams& p, uint64_t* bar, uint32_t parity) {
  if (!mbar_wait_bounded(bar, parity, kWaitNs)) {
    if ((threadIdx.x & 31) == 0) atomicOr(p.err, kErrTimeout);
  }
}

// An expert-table entry; the fields are clamped so that a corrupt table cannot address out of range.
struct ExpertInfo {
  int e, off, n;
  unsigned toks;
  float tsg, tsu, tsd;
};

// The expert table held by one warp in registers (lane l keeps entries l and l + 32), loaded once;
// an entry is then fetched by shuffles instead of a round trip to L2 per tile.
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

// ============================================================================================ gate|up

// gate|up shared memory: per warp a ring of 4 KB stages (16 rows x 256 B of codes, or 4 bf16 rows x
// 1 KB) and the scales of its current and next tile; per CTA the token rows of x (bf16, for the
// shared expert) and of the routed operand (int4: limbs, NVFP4: fp16), rows padded by 64 bytes so
// that the 8-lane phases of the fragment loads of different tokens hit different banks.
// Warps per CTA and stages per warp ring: int4 (at most 128 registers) runs 16 warps with 2 stages,
// NVFP4 (more registers per thread) 8 warps with 3; about 128 / 96 KB per SM in flight. A ring holds
// at most one tile's 4 stages, which keeps the scale double buffer safe.
template <int FMT>
struct GuGeom {
  static constexpr int kWarps = FMT == kInt4 ? 16 : 8;
  static constexpr int kDepth = FMT == kInt4 ? 2 : 3;
};
constexpr int kGuStage = 4096;
constexpr int kTokPitch = 2 * kH + 64;      // bytes per token row of x or of the routed operand

template <int FMT>
struct GuWarp {
  alignas(128) uint8_t stage[GuGeom<FMT>::kDepth][kGuStage];
  alignas(128) uint8_t scales[2][FMT == kInt4 ? 16 * (kH / kGroup) * 2 : 16 * (kH / 16)];
  uint64_t full[GuGeom<FMT>::kDepth];
};

template <int FMT>
struct GuShared {
  GuWarp<FMT> w[GuGeom<FMT>::kWarps];
  alignas(128) uint8_t xs[kDecodeMaxT][kTokPitch];    // x, bf16
  alignas(128) uint8_t xq[kDecodeMaxT][kTokPitch];    // int4: hi limbs, lo limbs; NVFP4: fp16 x
  float xsc[kDecodeMaxT][kH / kGroup];                // int4: unit / 16 of each segment of xq
  RouteSmem rs;
  uint64_t xbar;                                      // completion of the x copies
  uint64_t xqbar;                                     // completion of the operand copies
  uint64_t route_ready;                               // the routing warps have filled rs
};

// Warps kRouteWarp0.. of a gate|up CTA derive the routing (they hold no shared-expert tile: tile
// b + ncta * w is one only for w < 512 / ncta <= 4); the others wait for it on an mbarrier only when
// they reach a routed tile, so their shared-expert tiles never stall.
constexpr int kRouteWarp0 = 4;

// Warp-collective: stage s (K groups 4q..4q+3, q = s mod 4) of tile `tile`, as few large copies (the
// copy engine's cost is per copy more than per byte). Shared tile st: one tensor box with Sg rows
// 2st, 2st+1 and one with Su rows 2st, 2st+1 (1 KB each). Routed tile (gi, i8): one box of gate rows
// 8*i8 .. +8 and one of the matching up rows (256 B each); with q == 0 also the tile's scales.
template <int FMT>
__device__ void gu_issue(const DecodeParams& p, GuWarp<FMT>& ws, int s, int tile, const ExpertInfo& ex) {
  const int lane = threadIdx.x & 31;
  const int slot = s % GuGeom<FMT>::kDepth, q = s & 3;
  uint8_t* st = ws.stage[slot];
  uint64_t* bar = &ws.full[slot];
  if (tile < kShGuTiles) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 4 * 1024);
      tma_load_2d(st, &p.tm_sh_gu, q * 256, 2 * tile, bar);
      tma_load_2d(st + 2048, &p.tm_sh_gu, q * 256, kIs + 2 * tile, bar);
    }
    return;
  }
  const int i0 = 8 * ((tile - kShGuTiles) % kGuTilesPerExpert);
  const int erow = ex.e * (2 * kI);
  // scale bytes per row: int4 16 bf16 group scales, NVFP4 128 E4M3 block scales
  constexpr uint32_t row_sc = FMT == kInt4 ? (kH / kGroup) * 2 : kH / 16;
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, 16 * 256 + (q == 0 ? 16 * row_sc : 0));
    tma_load_2d(st, &p.tm_gu, q * 64, erow + i0, bar);
    tma_load_2d(st + 2048, &p.tm_gu, q * 64, erow + kI + i0, bar);
  }
  __syncwarp();
  if (q == 0 && (lane == 1 || lane == 2)) {        // gate rows' scales, then the up rows'
    uint8_t* sc = ws.scales[(s >> 2) & 1] + (lane - 1) * 8 * row_sc;
    bulk_g2s(sc, p.gu_scales + (static_cast<size_t>(erow) + (lane - 1) * kI + i0) * row_sc, 8 * row_sc, bar);
  }
}

// B operand of one group for one thread from a staged token row (32 stored elements, 64 bytes).
__device__ __forceinline__ void load_b_smem(RawB& B, const uint8_t* row, int j, int t, bool valid) {
  if (valid) {
    const uint8_t* p = row + (j * 128 + 32 * t) * 2;
#pragma unroll
    for (int q = 0; q < 4; ++q) B.u[q] = *reinterpret_cast<const uint4*>(p + 16 * q);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) B.u[q] = make_uint4(0, 0, 0, 0);
  }
}

// Limbs (hi row at row, lo row at row + kH) of a staged token row for group j: the thread's 32 bytes.
__device__ __forceinline__ void load_limbs_smem(uint4 (&bh)[2], uint4 (&bl)[2], const uint8_t* row, int j, int t,
                                                bool valid) {
  if (valid) {
    const uint8_t* ph = row + j * 128 + 32 * t;
    bh[0] = *reinterpret_cast<const uint4*>(ph);
    bh[1] = *reinterpret_cast<const uint4*>(ph + 16);
    bl[0] = *reinterpret_cast<const uint4*>(ph + kH);
    bl[1] = *reinterpret_cast<const uint4*>(ph + kH + 16);
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

template <int FMT>
__global__ void __launch_bounds__(GuGeom<FMT>::kWarps * 32, 1)
    decode_gate_up_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kWarps = GuGeom<FMT>::kWarps, kDepth = GuGeom<FMT>::kDepth;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  GuShared<FMT>& sm = *reinterpret_cast<GuShared<FMT>*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  GuWarp<FMT>& ws = sm.w[warp];
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < kDepth; ++i) mbar_init(&ws.full[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int ncta = gridDim.x;
  auto tile_of = [&](int k) { return static_cast<int>(blockIdx.x) + ncta * (warp + kWarps * k); };
  int na = -1;                                     // active experts; known after the grid dependency
  WarpTable tab;
  // Once per warp, the first time a routed tile is needed (or at the end). The routing warps wait
  // for the route kernel and derive the routing from its logits (CTA 0 also publishes the tables);
  // the first of them requests the operand rows and signals route_ready.
  auto routing = [&]() {
    if (na < 0) {
      if (warp >= kRouteWarp0) {
        pdl_wait();                                // the route kernel has finished and is visible
        route_group(p, sm.rs, blockIdx.x == 0, warp - kRouteWarp0, kWarps - kRouteWarp0, 1);
        // the down kernel reads CTA 0's published tables: they are visible before any trigger
        if (blockIdx.x == 0) __threadfence();
        pdl_trigger();
        if (warp == kRouteWarp0) {
          constexpr int kRow = 2 * kH;             // int4: hi + lo limbs; NVFP4: fp16
          const uint8_t* src = FMT == kInt4 ? p.xq8 : reinterpret_cast<const uint8_t*>(p.xq);
          if (lane == 0) mbar_arrive_expect_tx(&sm.xqbar, p.T * kRow + (FMT == kInt4 ? p.T * (kH / kGroup) * 4 : 0));
          __syncwarp();
          if (lane < p.T) bulk_g2s(sm.xq[lane], src + static_cast<size_t>(lane) * kRow, kRow, &sm.xqbar);
          if (FMT == kInt4 && lane == 31) bulk_g2s(&sm.xsc[0][0], p.xsc, p.T * (kH / kGroup) * 4, &sm.xqbar);
          if (lane == 0) mbar_arrive(&sm.route_ready);
        }
      } else {
        pdl_wait();
        wait_stage(p, &sm.route_ready, 0);
        pdl_trigger();
      }
      na = active_count(p, sm.rs);
      tab.load(sm.rs);
    }
  };
  auto valid = [&](int k) {                        // blocks until the routing is known if needed
    const int tl = tile_of(k);
    if (tl < kShGuTiles) return true;
    routing();
    return tl < kShGuTiles + kGuTilesPerExpert * na;
  };
  auto can_issue = [&](int k) {                    // as valid, but a shared-tile warp does not wait
    if (na < 0 && warp < kRouteWarp0 && tile_of(k) >= kShGuTiles && !mbar_test_wait(&sm.route_ready, 0))
      return false;
    return valid(k);
  };
  auto info = [&](int tl) {
    ExpertInfo ex{};
    if (tl >= kShGuTiles) ex = tab.get(p, (tl - kShGuTiles) / kGuTilesPerExpert);
    return ex;
  };

  // The shared expert's down weights need no routing either: into L2 now, in 32 KB chunks over the
  // CTAs, for the down kernel.
  if (threadIdx.x == 0)
    for (int c = blockIdx.x; c < kH * kIs * 2 / 32768; c += gridDim.x) prefetch_l2(p.sh_dn + c * 32768, 32768);
  // Shared-expert stages need no routing: request them first, then stage x and build the routed
  // operand while the route kernel runs.
  int s_issue = 0;
  for (; s_issue < kDepth && tile_of(s_issue >> 2) < kShGuTiles; ++s_issue)
    gu_issue(p, ws, s_issue, tile_of(s_issue >> 2), ExpertInfo{});
  if (warp == 0) {                                 // the token rows of x, one bulk copy each
    if (lane == 0) {
      mbar_init(&sm.xbar, 1);
      mbar_init(&sm.xqbar, 1);
      mbar_init(&sm.route_ready, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(&sm.xbar, p.T * kH * 2);
    }
    __syncwarp();
    if (lane < p.T) bulk_g2s(sm.xs[lane], p.x + static_cast<size_t>(lane) * kH, kH * 2, &sm.xbar);
  }
  __syncthreads();                                 // the barriers are initialised
  wait_stage(p, &sm.xbar, 0);
  bool have_xq = false;

  // the previous routed tile's segment arrival; the last arriver of a segment rotates it
  PendingArrival seg_arr;
  auto finish_last = [&](int key) {
    if (key < 0) return;
    const int gi = (key - kCntSeg) / 4, seg = (key - kCntSeg) % 4;
    finish_segment(p, tab.get(p, gi), seg);
    if (lane == 0) p.cnt[key] = 0;
  };
  float acc[2][4];
  ExpertInfo ex{};
  bool bvalid = false;
  int tok0 = 0, tok1 = 0;                          // tokens of MMA columns 2t, 2t+1
  const uint8_t* brow = nullptr;                   // this lane's activation row (column g)
  for (int s = 0;; ++s) {
    const int k = s >> 2, q = s & 3, tl = tile_of(k);
    if (q == 0 && !valid(k)) break;
    for (; s_issue < s + kDepth && can_issue(s_issue >> 2); ++s_issue)  // keep the ring full
      gu_issue(p, ws, s_issue, tile_of(s_issue >> 2), info(tile_of(s_issue >> 2)));
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
        brow = sm.xq[bvalid ? token_of(p, ex, g) : 0];
      }
    }
    const int slot = s % kDepth;
    wait_stage(p, &ws.full[slot], (s / kDepth) & 1);
    const uint8_t* st = ws.stage[slot];
    if (tl < kShGuTiles) {
      // rows g = 0,1: gate 2tl, 2tl+1; g = 2,3: up 2tl, 2tl+1; MMA rows 4..15 are zero
      const bool xv = g < p.T;
      const uint8_t* xr = sm.xs[xv ? g : 0];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        RawA<kBf16> A;
        load_a_bf16_rows(A, st, 1024, 4, g, jj, t);
        RawB B;
        load_b_smem(B, xr, 4 * q + jj, t, xv);
        bf16_group(acc, A, B, nullptr);
      }
    } else if constexpr (FMT == kInt4) {
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(ws.scales[k & 1]);
      const bool v0 = 2 * t < ex.n, v1 = 2 * t + 1 < ex.n;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * q + jj;
        const uint4 ra = *reinterpret_cast<const uint4*>(st + g * 256 + jj * 64 + 16 * t);
        const uint4 rb = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + jj * 64 + 16 * t);
        uint4 bh[2], bl[2];
        load_limbs_smem(bh, bl, brow, j, t, bvalid);
        const float sg = bf16_bits_to_f32(sc[g * 16 + j]), su = bf16_bits_to_f32(sc[(8 + g) * 16 + j]);
        const float x0 = v0 ? sm.xsc[tok0][j] : 0.f, x1 = v1 ? sm.xsc[tok1][j] : 0.f;
        const float f[4] = {sg * x0, sg * x1, su * x0, su * x1};
        int4_group(acc[0], ra, rb, bh, bl, f);
      }
    } else {
      const uint8_t* sc = ws.scales[k & 1];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * q + jj;
        const uint4 ra = *reinterpret_cast<const uint4*>(st + g * 256 + jj * 64 + 16 * t);
        const uint4 rb = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + jj * 64 + 16 * t);
        RawB B;
        load_b_smem(B, brow, j, t, bvalid);
        nvfp4_group(acc, ra, rb, B, sc + g * 128, sc + 1024 + g * 128, j, t);
      }
    }
    __syncwarp();                                  // every lane's reads of the slot precede its refill
    if (q != 3) continue;
    // ---- tile epilogue
    float c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = acc[0][i] + acc[1][i];
    if (tl < kShGuTiles) {
      const float u0 = __shfl_down_sync(kFull, c[0], 8), u1 = __shfl_down_sync(kFull, c[1], 8);
      if (g < 2) {
        const float uv[2] = {u0, u1};
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int tok = 2 * t + qq;
          if (tok < p.T) {
            const float hs = silu(c[qq]) * uv[qq];
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
          p.h32[static_cast<size_t>(ex.off + col) * kI + 8 * i8 + g] = silu(c[qq] * ex.tsg) * (c[2 + qq] * ex.tsu);
      }
      const int seg = i8 / (kGroup / 8);
      finish_last(seg_arr.settle());
      seg_arr.arrive(p.cnt, kCntSeg + 4 * gi + seg, kGroup / 8);
    }
  }
  routing();                                       // every warp passes the grid dependency before it ends
  finish_last(seg_arr.settle());
  if (!have_xq) wait_stage(p, &sm.xqbar, 0);       // no bulk copy may still write this CTA's memory
}

// ============================================================================================ down

// Warp-collective: stage q of tile `tile` (slot s mod depth). Shared tile sd: one tensor box with
// Sd rows 8sd .. +8, K quarter q (512 B each). Routed tile (gi, b): 16 rows 32b + 16q .. +16 of the
// expert's down rows, all of K (256 B each, contiguous), and their scales.
template <int FMT>
__device__ void dn_issue(const DecodeParams& p, DnWarp<FMT>& ws, int s, int q, int tile, const ExpertInfo& ex) {
  const int lane = threadIdx.x & 31;
  const int slot = s % DnGeom<FMT>::kDepth;
  uint8_t* st = ws.stage[slot];
  uint64_t* bar = &ws.full[slot];
  if (tile < kShDnTiles) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 4096);
      tma_load_2d(st, &p.tm_sh_dn, q * 128, 8 * tile, bar);
    }
    return;
  }
  const int n0 = 32 * ((tile - kShDnTiles) % kDnTilesPerExpert) + 16 * q;
  const size_t row0 = static_cast<size_t>(ex.e) * kH + n0;
  // scale bytes per row: int4 4 bf16 group scales, NVFP4 32 E4M3 block scales
  const uint32_t row_sc = p.fmt == kInt4 ? (kI / kGroup) * 2 : kI / 16;
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, 4096 + 16 * row_sc);
    bulk_g2s(st, p.dn_codes + row0 * (kI / 2), 4096, bar);
    bulk_g2s(st + 4096, p.dn_scales + row0 * row_sc, 16 * row_sc, bar);
  }
}

__device__ __forceinline__ void prefetch_l1(const void* ptr) { asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr)); }

// Warp: brings `bytes` bytes at base into this SM's L1, one 128-byte line per lane and step.
__device__ __forceinline__ void prefetch_range(const void* base, size_t bytes) {
  const uint8_t* b = static_cast<const uint8_t*>(base);
  for (size_t o = static_cast<size_t>(threadIdx.x & 31) * 128; o < bytes; o += 32 * 128) prefetch_l1(b + o);
}

// Warp: L1 prefetch of the activation rows a shared down tile reads (hs of every token; call after
// the grid dependency). Routed tiles read their operand from shared memory.
__device__ void dn_prefetch(const DecodeParams& p, int tile, const ExpertInfo&) {
  if (tile < kShDnTiles) {
    prefetch_range(p.hs_hi, static_cast<size_t>(p.T) * kIs * 2);
    prefetch_range(p.hs_lo, static_cast<size_t>(p.T) * kIs * 2);
  }
}

// y rows nb*64 .. +64 of every token (one warp), slots in slot order. The (position, weight) of
// every pair is fetched once (lane q holds pairs q and q + 32); lane l then owns rows 4(l mod 16)
// .. +4 of token t0 + l/16, two tokens per round.
__device__ void combine_block(const DecodeParams& p, const RouteSmem& rs, int nb) {
  const int lane = threadIdx.x & 31;
  const int n = nb * 64 + 4 * (lane & 15), K = p.K, P = p.T * K;
  int pos[2];
  float wt[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = lane + 32 * h;
    pos[h] = q < P ? min(max(rs.inv[q], 0), P - 1) : 0;
    wt[h] = q < P ? rs.w[q] : 0.f;
  }
#pragma unroll 1
  for (int t0 = 0; t0 < p.T; t0 += 2) {
    const int tok = t0 + (lane >> 4);
    const bool tv = tok < p.T;
    const float4 yv = tv ? __ldcg(reinterpret_cast<const float4*>(p.ys + tok * kH + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 ov[kMaxTopK];
    float w[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      if (k < K) {
        const int q = min(tok, p.T - 1) * K + k;         // per lane: read both halves of the table
        const int p0 = __shfl_sync(kFull, pos[0], q & 31), p1 = __shfl_sync(kFull, pos[1], q & 31);
        const float w0 = __shfl_sync(kFull, wt[0], q & 31), w1 = __shfl_sync(kFull, wt[1], q & 31);
        w[k] = q < 32 ? w0 : w1;
        ov[k] = tv ? __ldcg(reinterpret_cast<const float4*>(p.o + static_cast<size_t>(q < 32 ? p0 : p1) * kH + n))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (tv) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k)
        if (k < K) {
          a[0] = fmaf(w[k], ov[k].x, a[0]);
          a[1] = fmaf(w[k], ov[k].y, a[1]);
          a[2] = fmaf(w[k], ov[k].z, a[2]);
          a[3] = fmaf(w[k], ov[k].w, a[3]);
        }
      uint2 out;
      out.x = pack_bf162(fmaf(p.routed_scale, a[0], yv.x), fmaf(p.routed_scale, a[1], yv.y));
      out.y = pack_bf162(fmaf(p.routed_scale, a[2], yv.z), fmaf(p.routed_scale, a[3], yv.w));
      *reinterpret_cast<uint2*>(p.y + tok * kH + n) = out;
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(DnGeom<FMT>::kWarps * 32, 1)
    decode_down_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int kWarps = DnGeom<FMT>::kWarps, kDepth = DnGeom<FMT>::kDepth;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  DnShared<FMT>& sm = *reinterpret_cast<DnShared<FMT>*>(smem_raw);
  DnWarp<FMT>& ws = sm.w[warp];
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < kDepth; ++i) mbar_init(&ws.full[i], 1);
    if (warp == 0) mbar_init(&sm.hqbar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  // This kernel starts only after every gate|up warp has triggered, and gate|up CTA 0 triggers only
  // after publishing the routing tables (fenced): they are read here while gate|up still runs. The
  // gate|up outputs are read only after pdl_wait below.
  if (warp == 0) {
    const int nact = min(max(__ldcg(p.n_active), 0), min(kMaxActive, p.T * p.K));
    for (int gi = lane; gi < nact; gi += 32) {
      sm.rs.etab[gi][0] = __ldcg(p.etab + 2 * gi);
      sm.rs.etab[gi][1] = __ldcg(p.etab + 2 * gi + 1);
    }
    for (int q = lane; q < p.T * p.K; q += 32) {
      sm.rs.inv[q] = __ldcg(p.inv + q);
      sm.rs.w[q] = __ldcg(p.wts + q);
    }
    if (lane == 0) sm.rs.na = nact;
  }
  __syncthreads();
  const int na = active_count(p, sm.rs);
  WarpTable tab;
  tab.load(sm.rs);
  const int n_tiles = kShDnTiles + kDnTilesPerExpert * na;
  const int ncta = gridDim.x;
  auto tile_of = [&](int k) { return static_cast<int>(blockIdx.x) + ncta * (warp + kWarps * k); };
  auto info = [&](int tl) {
    ExpertInfo ex{};
    if (tl >= kShDnTiles) ex = tab.get(p, (tl - kShDnTiles) / kDnTilesPerExpert);
    return ex;
  };
  // Stage s of this warp -> (tile ordinal k, stage q in the tile): a shared tile has 4 stages and can
  // only be a warp's first tile (ncta * kWarps > kShDnTiles), routed tiles have 2.
  const int first_len = tile_of(0) < kShDnTiles ? 4 : 2;
  auto stage_k = [&](int s) { return s < first_len ? 0 : 1 + (s - first_len) / 2; };
  auto stage_q = [&](int s) { return s < first_len ? s : (s - first_len) % 2; };
  auto issue = [&](int s) {
    const int tl = tile_of(stage_k(s));
    dn_issue<FMT>(p, ws, s, stage_q(s), tl, info(tl));
  };
  int s_issue = 0;
  for (; s_issue < kDepth && tile_of(stage_k(s_issue)) < n_tiles; ++s_issue) issue(s_issue);
  pdl_wait();                                      // h and hs of the gate|up kernel
  if (warp == 0 && lane == 0) {                    // the down operand of every position, one copy
    const int P = p.T * p.K;
    mbar_arrive_expect_tx(&sm.hqbar, P * 2 * kI + (FMT == kInt4 ? P * (kI / kGroup) * 4 : 0));
    bulk_g2s(&sm.hq[0][0], FMT == kInt4 ? p.hq8 : reinterpret_cast<const uint8_t*>(p.hq), P * 2 * kI, &sm.hqbar);
    if (FMT == kInt4) bulk_g2s(&sm.hsc[0][0], p.hsc, P * (kI / kGroup) * 4, &sm.hqbar);
  }
  bool have_hq = false;
  if (tile_of(0) < n_tiles) dn_prefetch(p, tile_of(0), info(tile_of(0)));

  // the previous tile's block arrival; the last arriver of a 64-row block combines it
  PendingArrival blk_arr;
  auto combine_last = [&](int key) {
    if (key < 0) return;
    combine_block(p, sm.rs, key - kCntBlk);
    if (lane == 0) p.cnt[key] = 0;
  };
  float acc[2][2][4];                              // [16-row half][accumulator set][fragment]
  ExpertInfo ex{};
  const int target = 2 * na + kShDnTiles / (kH / 64);
  for (int s = 0;; ++s) {
    const int k = stage_k(s), q = stage_q(s), tl = tile_of(k);
    if (tl >= n_tiles) break;
    if (q == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][0][i] = acc[h][1][i] = 0.f;
      if (tl >= kShDnTiles) ex = info(tl);
      if (tile_of(k + 1) < n_tiles) dn_prefetch(p, tile_of(k + 1), info(tile_of(k + 1)));
    }
    const int slot = s % kDepth;
    wait_stage(p, &ws.full[slot], (s / kDepth) & 1);
    const uint8_t* st = ws.stage[slot];
    if (tl < kShDnTiles) {
      // rows 8tl + g (g < 8) of Sd, K quarter q (groups 2q, 2q+1); hs as a bf16 pair (hi + lo)
      const bool bv = g < p.T;
      const size_t r = static_cast<size_t>(bv ? g : 0) * kIs;
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        RawA<kBf16> A;
        load_a_bf16_rows(A, st, 512, 8, g, jj, t);
        RawB Bh, Bl;
        Bh.load(p.hs_hi + r, 2 * q + jj, t, bv);
        Bl.load(p.hs_lo + r, 2 * q + jj, t, bv);
        bf16_group(acc[0], A, Bh, &Bl);
      }
    } else {
      // 16 rows (half q of the 32-row tile), all of K = 4 groups
      if (!have_hq) {
        wait_stage(p, &sm.hqbar, 0);
        have_hq = true;
      }
      const bool bv = g < ex.n;
      const uint8_t* hrow = sm.hq[ex.off + (bv ? g : 0)];
      const uint8_t* sc = st + 4096;
      if constexpr (FMT == kInt4) {
        const uint16_t* s16 = reinterpret_cast<const uint16_t*>(sc);
        const bool v0 = 2 * t < ex.n, v1 = 2 * t + 1 < ex.n;
        const float* x0p = sm.hsc[ex.off + (v0 ? 2 * t : 0)];
        const float* x1p = sm.hsc[ex.off + (v1 ? 2 * t + 1 : 0)];
#pragma unroll
        for (int j = 0; j < kI / kGroup; ++j) {
          const uint4 ra = *reinterpret_cast<const uint4*>(st + g * 256 + j * 64 + 16 * t);
          const uint4 rb = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + j * 64 + 16 * t);
          uint4 bh[2], bl[2];
          if (bv) {
            const uint8_t* ph = hrow + j * 128 + 32 * t;
            bh[0] = *reinterpret_cast<const uint4*>(ph);
            bh[1] = *reinterpret_cast<const uint4*>(ph + 16);
            bl[0] = *reinterpret_cast<const uint4*>(ph + kI);
            bl[1] = *reinterpret_cast<const uint4*>(ph + kI + 16);
          } else {
            bh[0] = bh[1] = bl[0] = bl[1] = make_uint4(0, 0, 0, 0);
          }
          const float s0 = bf16_bits_to_f32(s16[g * 4 + j]), s1 = bf16_bits_to_f32(s16[(g + 8) * 4 + j]);
          const float x0 = v0 ? x0p[j] : 0.f, x1 = v1 ? x1p[j] : 0.f;
          const float f[4] = {s0 * x0, s0 * x1, s1 * x0, s1 * x1};
          int4_group(acc[q][0], ra, rb, bh, bl, f);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kI / kGroup; ++j) {
          const uint4 ra = *reinterpret_cast<const uint4*>(st + g * 256 + j * 64 + 16 * t);
          const uint4 rb = *reinterpret_cast<const uint4*>(st + (g + 8) * 256 + j * 64 + 16 * t);
          RawB B;
          load_b_smem(B, hrow, j, t, bv);
          nvfp4_group(acc[q], ra, rb, B, sc + g * 32, sc + (g + 8) * 32, j, t);
        }
      }
    }
    __syncwarp();                                  // every lane's reads of the slot precede its refill
    if (tile_of(stage_k(s_issue)) < n_tiles) {     // s_issue == s + kDepth: refill this slot
      issue(s_issue);
      ++s_issue;
    }
    if (q != (tl < kShDnTiles ? 3 : 1)) continue;
    // ---- tile epilogue
    int nb;
    if (tl < kShDnTiles) {
      const int n0 = 8 * tl;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int tok = 2 * t + qq;
        if (tok < p.T) p.ys[tok * kH + n0 + g] = acc[0][0][qq] + acc[0][1][qq];
      }
      nb = n0 / 64;
    } else {
      const int b = (tl - kShDnTiles) % kDnTilesPerExpert;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int col = 2 * t + (qq & 1);
          if (col < ex.n)
            p.o[static_cast<size_t>(ex.off + col) * kH + 32 * b + 16 * h + g + 8 * (qq >> 1)] =
                (acc[h][0][qq] + acc[h][1][qq]) * ex.tsd;
        }
      nb = b / 2;
    }
    combine_last(blk_arr.settle());
    blk_arr.arrive(p.cnt, kCntBlk + nb, target);
  }
  combine_last(blk_arr.settle());
  if (!have_hq) wait_stage(p, &sm.hqbar, 0);       // no bulk copy may still write this CTA's memory
}

template <typename Kern>
cudaError_t launch_ex(Kern kernel, int grid, int threads, size_t smem, bool pdl, cudaStream_t s,
                      const DecodeParams& p) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Dynamic shared memory limit, and the same L1/shared split for every decode kernel so that an SM
// need not be reconfigured between them.
template <typename Kern>
cudaError_t allow_smem(Kern kernel, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int n_sm, cudaStream_t s, cudaEvent_t ev_after_route,
                          cudaEvent_t ev_after_gate_up) {
  constexpr size_t kGuSmem4 = sizeof(GuShared<kInt4>), kGuSmemF = sizeof(GuShared<kNvfp4>);
  constexpr size_t kDnSmem4 = sizeof(DnShared<kInt4>), kDnSmemF = sizeof(DnShared<kNvfp4>);
  static_assert(kGuSmem4 <= 227 * 1024 && kGuSmemF <= 227 * 1024 && kDnSmem4 <= 227 * 1024 && kDnSmemF <= 227 * 1024,
                "shared memory per CTA");
  static bool smem_set = false;                    // per process; the attribute is per function
  if (!smem_set) {
    cudaError_t e;
    if ((e = allow_smem(decode_gate_up_kernel<kInt4>, kGuSmem4)) != cudaSuccess) return e;
    if ((e = allow_smem(decode_gate_up_kernel<kNvfp4>, kGuSmemF)) != cudaSuccess) return e;
    if ((e = allow_smem(decode_down_kernel<kInt4>, kDnSmem4)) != cudaSuccess) return e;
    if ((e = allow_smem(decode_down_kernel<kNvfp4>, kDnSmemF)) != cudaSuccess) return e;
    if ((e = allow_smem(decode_route_kernel, 0)) != cudaSuccess) return e;
    smem_set = true;
  }
  cudaError_t e = launch_ex(decode_route_kernel, (p.E + kRouteWarps - 1) / kRouteWarps, kRouteWarps * 32, 0, false,
                            s, p);
  if (e != cudaSuccess) return e;
  if (ev_after_route && (e = cudaEventRecord(ev_after_route, s)) != cudaSuccess) return e;
  e = p.fmt == kInt4 ? launch_ex(decode_gate_up_kernel<kInt4>, n_sm, GuGeom<kInt4>::kWarps * 32, kGuSmem4, true, s, p)
                     : launch_ex(decode_gate_up_kernel<kNvfp4>, n_sm, GuGeom<kNvfp4>::kWarps * 32, kGuSmemF, true, s, p);
  if (e != cudaSuccess) return e;
  if (ev_after_gate_up && (e = cudaEventRecord(ev_after_gate_up, s)) != cudaSuccess) return e;
  return p.fmt == kInt4 ? launch_ex(decode_down_kernel<kInt4>, n_sm, DnGeom<kInt4>::kWarps * 32, kDnSmem4, true, s, p)
                        : launch_ex(decode_down_kernel<kNvfp4>, n_sm, DnGeom<kNvfp4>::kWarps * 32, kDnSmemF, true, s, p);
}

}  // namespace flint
