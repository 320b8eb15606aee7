// Device-side helpers shared by the Flint MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace flint {

// Programmatic dependent launch: the next kernel of the stream may be scheduled once every CTA of this
// one has called launch_dependents (or exited); wait blocks until the previous kernel has completed
// and its writes are visible (a no-op without a programmatic predecessor).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kH = 2048;        // hidden width
constexpr int kI = 512;         // routed SwiGLU width
constexpr int kIs = 1024;       // shared-expert SwiGLU width
constexpr int kGroup = 128;     // int4 scale group and Hadamard width
constexpr int kMaxTopK = 8;
constexpr int kMaxE = 256;

enum WFmt : int { kInt4 = 0, kNvfp4 = 1, kBf16 = 2 };

// error word bits
constexpr unsigned kErrBadId = 1u << 0;
constexpr unsigned kErrBadOffset = 1u << 1;
constexpr unsigned kErrTimeout = 1u << 2;
constexpr unsigned kErrRange = 1u << 3;

// --------------------------------------------------------------------------------------------
// loads

// 16-byte streaming load of read-only data that is used once (weights): do not keep it in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16-byte read-only load that may hit in L1 (activations reused by many warps).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  return __ldg(reinterpret_cast<const uint2*>(p));
}

// 16-byte load through L2 only (data written earlier in the same kernel by other CTAs).
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  return __ldcg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Fire-and-forget add with release semantics at GPU scope (publishes the writes that precede it,
// including other CTA threads' writes ordered before it by a barrier).
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// --------------------------------------------------------------------------------------------
// shared-memory barriers and bulk copies (sm_90+)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Like mbar_try_wait, but the thread may sleep until the phase completes or about `hint_ns`
// nanoseconds pass, instead of polling: waiting warps then take no issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a barrier phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void red_relaxed_add(int* p, int v) {
  asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

constexpr uint32_t kWaitSleepNs = 20000;      // longest sleep of a bounded wait between clock checks

// Waits for the barrier phase with the given parity; gives up after `limit_ns` and returns false.
// The clock is read every 16th poll only, so that waiting warps take few issue slots from working
// ones.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (unsigned i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if ((i & 15u) == 0u && globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Bulk copy global -> this CTA's shared memory, completing `bytes` of transaction on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Orders this thread's earlier generic-proxy observations (e.g. an acquire of data other CTAs wrote)
// before its later bulk-copy (async-proxy) reads of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also returns the OR of `pred` over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// --------------------------------------------------------------------------------------------
// number formats

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b),
                      *reinterpret_cast<__half2*>(&c));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t mask, uint32_t x) {
  // (a & mask) ^ x in one instruction
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(a), "r"(mask), "r"(x));
  return r;
}

// int4 (two's complement) -> fp16 pairs. A 32-bit word holds eight codes n0..n7 (n0 in bits 0..3).
// The four results are the exact fp16 pairs (n0,n4), (n1,n5), (n2,n6), (n3,n7) (low half first):
// codes are turned into offset binary u = n ^ 8 inside an fp16 of value 1024+u (or 1024+16u for
// the odd nibbles) and rebased with one exact fused multiply-add.
__device__ __forceinline__ void int4x8_to_half2x4(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t kLoMagic = 0x64086408u;   // 0x6400 | bit 3 flipped  (value 1024 + u)
  const uint32_t kHiMagic = 0x64806480u;   // 0x6400 | bit 7 flipped  (value 1024 + 16u)
  const uint32_t kOne = 0x3C003C00u;       // 1.0
  const uint32_t kSixteenth = 0x2C002C00u; // 1/16
  const uint32_t kNeg1032 = 0xE408E408u;   // -1032
  const uint32_t kNeg72 = 0xD480D480u;     // -72
  uint32_t w8 = w >> 8;
  p[0] = hfma2_u32(lop3_and_xor(w, 0x000F000Fu, kLoMagic), kOne, kNeg1032);
  p[1] = hfma2_u32(lop3_and_xor(w, 0x00F000F0u, kHiMagic), kSixteenth, kNeg72);
  p[2] = hfma2_u32(lop3_and_xor(w8, 0x000F000Fu, kLoMagic), kOne, kNeg1032);
  p[3] = hfma2_u32(lop3_and_xor(w8, 0x00F000F0u, kHiMagic), kSixteenth, kNeg72);
}

// Two E2M1 codes (one byte, low nibble first) -> fp16 pair, by the hardware conversion.
__device__ __forceinline__ uint32_t e2m1x2_to_half2(uint32_t byte) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte & 0xFFu), __NV_E2M1);
  return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// One E4M3 (fn) byte -> fp16 bits (exact).
__device__ __forceinline__ uint16_t e4m3_to_half_bits(uint32_t byte) {
  __half_raw r = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte & 0xFFu), __NV_E4M3);
  return r.x;
}

// --------------------------------------------------------------------------------------------
// warp-level tensor-core dot products (m16n8k16, fp32 accumulate)

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// --------------------------------------------------------------------------------------------
// 128-wide Walsh-Hadamard transform of one segment held by a warp: lane l holds the naturally
// ordered elements 4l..4l+3. Butterflies in registers for distances 1 and 2 and across lanes for
// 4..64; the result is scaled by 1/sqrt(128), so applying it twice is the identity.
__device__ __forceinline__ void fwht128_warp(float (&v)[4]) {
  float a, b;
  a = v[0]; b = v[1]; v[0] = a + b; v[1] = a - b;
  a = v[2]; b = v[3]; v[2] = a + b; v[3] = a - b;
  a = v[0]; b = v[2]; v[0] = a + b; v[2] = a - b;
  a = v[1]; b = v[3]; v[1] = a + b; v[3] = a - b;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float o = __shfl_xor_sync(0xFFFFFFFFu, v[j], m);
      v[j] = upper ? (o - v[j]) : (v[j] + o);
    }
  }
  const float kInvSqrt128 = 0.08838834764831845f;
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] *= kInvSqrt128;
}

// Stores the four values of lane l (natural elements 4l..4l+3 of a 128-segment) as fp16 into
// `dst` (the segment's first element), either in natural order or with every 8-block in the
// order 0,4,1,5,2,6,3,7 (the order the int4 decoder produces its fp16 pairs in).
__device__ __forceinline__ void store_seg_half(__half* dst, const float (&v)[4], bool pair_order) {
  const int lane = threadIdx.x & 31;
  if (!pair_order) {
    uint2 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    *reinterpret_cast<uint2*>(dst + 4 * lane) = u;
    return;
  }
  // 8-block b = lane/2 holds natural a0..a3 (even lane) and b0..b3 (odd lane); stored order is
  // a0 b0 a1 b1 | a2 b2 a3 b3, so the even lane writes the first half and the odd lane the second.
  const bool odd = lane & 1;
  float s0 = odd ? v[0] : v[2];
  float s1 = odd ? v[1] : v[3];
  float r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
  float r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
  uint2 u;
  if (!odd) {            // a0 b0 a1 b1
    u.x = pack_half2(v[0], r0);
    u.y = pack_half2(v[1], r1);
  } else {               // a2 b2 a3 b3  (r0,r1 = a2,a3 from the even partner)
    u.x = pack_half2(r0, v[2]);
    u.y = pack_half2(r1, v[3]);
  }
  *reinterpret_cast<uint2*>(dst + 8 * (lane >> 1) + 4 * (lane & 1)) = u;
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

}  // namespace flint
