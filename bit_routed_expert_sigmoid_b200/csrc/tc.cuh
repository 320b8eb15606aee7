// Primitives of the tcgen05 grouped-GEMM kernels (prefill): tensor-memory MMA and copies, TMA tile
// loads, bounded mbarrier waits, and the tile table that walks the routed experts' permuted rows.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace flint {

namespace {

#ifndef FLINT_WAIT_NS
#define FLINT_WAIT_NS 1000000000ull          // 1 s
#endif
constexpr uint64_t kPfWaitNs = FLINT_WAIT_NS;
constexpr unsigned kAll = 0xFFFFFFFFu;

constexpr int kPfN = 64;                     // tokens per tile (MMA N, padded to a multiple of 16)

// ---------------------------------------------------------------------------------------------
// tcgen05 / TMA primitives

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Warp-wide MMA and commit: every lane of the warp executes the call with the same operands (so they can stay
// in uniform registers) and one elected lane issues the instruction.
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_mma_ta_w(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void tc_mma_ss_w(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
}

// 32 consecutive columns of the warp's 32 lanes (lane i of the warp = its own row)
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16 with fp32 D, K-major A and B, M = 128.
__device__ __forceinline__ uint32_t idesc_m128(int n, bool bf16) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// L2 policy for data a kernel reads exactly once (the weights): its lines are evicted first, so that
// what the next kernels read again (activations, h, o) stays in L2.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tma_2d_hint(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3}], "
      "[%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Bounded wait: false if the CTA has given up (another wait expired) or this one expires.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kPfWaitNs) {
      atomicOr(err, kErrTimeout);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// Every lane waits (each acquires the barrier's phase itself); the verdict is warp-uniform.
__device__ __forceinline__ bool pf_wait_all(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned* err) {
  const bool ok = pf_wait(bar, parity, abort, err);
  return __all_sync(kAll, ok) != 0;
}

// ---------------------------------------------------------------------------------------------
// tile table of the routed kernels

struct TileTab {
  int n, total;
  int start[kMaxE + 1];   // first tile of expert i
  int e[kMaxE];
  int w[kMaxE];           // weight index of expert i: its slot when the weights sit in cache slots, else i
  int off[kMaxE];         // first permuted row
  int cnt[kMaxE];         // permuted rows
  int nch[kMaxE];         // chunks of kPfN rows
  int cbase[kMaxE];       // index of expert i's first chunk among all experts' chunks (ascending expert)
};

struct PfTile {
  int e, w, row0, n, rp;  // expert, its weight index, first permuted row of the chunk, rows in it (1..kPfN), block pair
  int c;                  // chunk index (cbase of the expert + chunk)
};

// Warp 0: tiles of expert e are rp-major over its chunks; experts in ascending order (an expert
// without rows has none). Every lane loads the offsets (and weight slots) of all its experts before
// the scans, so the table costs one global-load latency rather than one per 32 experts. kChunks:
// also number every expert's chunks (cbase; only the W4A4 kernels address data by chunk).
template <bool kChunks>
__device__ void build_tiles(TileTab& tt, const PrefillParams& p, int rp_count) {
  constexpr int kPer = kMaxE / 32;
  const int lane = threadIdx.x & 31;
  const int n = min(p.E, kMaxE);
  int off[kPer], end[kPer], slot[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = 32 * j + lane;
    off[j] = i < n ? __ldg(p.offsets + i) : 0;
    end[j] = i < n ? __ldg(p.offsets + i + 1) : 0;
    slot[j] = (i < n && p.slot_of) ? __ldg(p.slot_of + i) : i;
  }
  int base = 0, cb = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = 32 * j + lane;
    int tiles = 0, nchunks = 0;
    if (i < n) {
      const int c = max(end[j] - off[j], 0);
      const int nch = (c + kPfN - 1) / kPfN;
      tt.e[i] = i;
      tt.w[i] = (p.slot_of && c > 0) ? min(max(slot[j], 0), p.n_wslots - 1) : i;
      tt.off[i] = off[j];
      tt.cnt[i] = c;
      tt.nch[i] = nch;
      tiles = rp_count * nch;
      nchunks = nch;
    }
    int v = tiles, vc = nchunks;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(kAll, v, d), uc = __shfl_up_sync(kAll, vc, d);
      if (lane >= d) {
        v += u;
        vc += uc;
      }
    }
    if (i < n) {
      tt.start[i] = base + v - tiles;
      if constexpr (kChunks) tt.cbase[i] = cb + vc - nchunks;
    }
    base += __shfl_sync(kAll, v, 31);
    cb += __shfl_sync(kAll, vc, 31);
  }
  if (lane == 0) {
    tt.n = n;
    tt.total = base;
    tt.start[n] = base;
  }
}

template <bool kChunks>
__device__ __forceinline__ PfTile tile_at(const TileTab& tt, int t) {
  int lo = 0, hi = tt.n - 1;                 // last i with start[i] <= t (t < total)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tt.start[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int local = t - tt.start[lo], nch = tt.nch[lo];
  const int rp = local / nch, ch = local - rp * nch;
  PfTile r;
  r.e = tt.e[lo];
  r.w = tt.w[lo];
  r.row0 = tt.off[lo] + ch * kPfN;
  r.n = min(kPfN, tt.cnt[lo] - ch * kPfN);
  r.rp = rp;
  r.c = kChunks ? tt.cbase[lo] + ch : 0;
  return r;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// silu with the fast exponential and division (relative error a few ulp of fp32)
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

}  // namespace

}  // namespace flint
