// Routing stage of the prefill path of the Flint MoE layer: unbiased sigmoid top-k with the
// selected-sum floor, the expert-major permutation of (token, slot) pairs, and the activation
// operand of the routed experts (x rotated per 128-segment for the int4 format). The forward's
// router logits come from the tensor-core kernel in prefill.cu; the CUDA-core kernel here serves the
// routing-only entry point.
#include "kernels.cuh"

namespace flint {

// ---------------------------------------------------------------------------------------------
// Router logits on CUDA cores, for the routing-only entry point (small T): logits[t][e] = sum_j W_r[e][j] * x[t][j]. The bf16 x bf16 products
// are exact in fp32 and accumulate in fp32 (the router rows are used widened to FP32 on the
// pages: WaveCut/Flint-UD-Q4_K_XL-NInfer-v3, "What is inside"). One warp owns one expert row and
// a chunk of up to 8 tokens; lane l covers elements 8l + 256i (i = 0..7) so every load is a
// coalesced 16-byte access.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ wr, int T, int E,
                                                            float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  const int t0 = blockIdx.y * 8;
  if (e >= E) return;
  const int nt = min(8, T - t0);
  uint4 wv[8];
  const uint16_t* wrow = wr + static_cast<size_t>(e) * kH;
#pragma unroll
  for (int i = 0; i < 8; ++i) wv[i] = ld_nc_v4(wrow + 8 * lane + 256 * i);
  float acc[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t] = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    if (t < nt) {
      const uint16_t* xr = x + static_cast<size_t>(t0 + t) * kH;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 xv = ld_nc_v4(xr + 8 * lane + 256 * i);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[t] = fmaf(bf16lo_to_f32(xw[q]), bf16lo_to_f32(ww[q]), acc[t]);
          acc[t] = fmaf(bf16hi_to_f32(xw[q]), bf16hi_to_f32(ww[q]), acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    float v = acc[t];
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, m);
    if (lane == 0 && t < nt) logits[static_cast<size_t>(t0 + t) * E + e] = v;
  }
}

// ---------------------------------------------------------------------------------------------
// Top-k selection, one warp per token. The router is unbiased (midagedev/bloomery issue #632,
// design-round comment), so the k largest sigmoid scores are the k largest logits (sigmoid is
// strictly increasing); selecting on the fp32 logits avoids the ties fp32 sigmoid saturation
// would create. Ties go to the lower expert id. The chosen slots are listed by ascending expert
// id, and w_k = s_k / max(sum of the chosen s, floor) with s = sigmoid(logit) (the SelectedSumFloor
// policy, same issue, host-policy comment). The sum runs in slot order.
template <int NS>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   float* __restrict__ logits_out, int T, int E, int K,
                                                   float floor_, int* __restrict__ ids, float* __restrict__ wts,
                                                   unsigned flags, unsigned* __restrict__ err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const int per = E >> 5;          // logits per lane (E is a multiple of 32, at most 256)
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float part[NS];
#pragma unroll
    for (int q = 0; q < NS; ++q)
      part[q] = (j < per) ? __ldg(logits + static_cast<size_t>(q) * T * E + static_cast<size_t>(t) * E + lane + 32 * j)
                          : 0.f;
    float a = part[0];
#pragma unroll
    for (int q = 1; q < NS; ++q) a += part[q];     // slice order
    v[j] = (j < per) ? a : -INFINITY;
  }
  if (logits_out) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per) logits_out[static_cast<size_t>(t) * E + lane + 32 * j] = v[j];
  }
  unsigned taken = 0;              // bit j: element lane+32j already chosen
  int my_id = 0x7FFFFFFF;          // lane k < K: the k-th pick
  float my_l = 0.f;
  for (int k = 0; k < K; ++k) {
    // local best: highest logit, then lowest index
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int idx = lane + 32 * j;
      const bool ok = (j < per) && !((taken >> j) & 1u);
      if (ok && (v[j] > bv || (v[j] == bv && idx < bi))) { bv = v[j]; bi = idx; }
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, m);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, m);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == k) {
      my_id = bi;
      my_l = bv;
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
  }
  // slot of the pick = its rank by expert id; lane r then takes the pick of rank r
  int rank = 0;
  for (int j = 0; j < K; ++j) rank += (__shfl_sync(0xFFFFFFFFu, my_id, j) < my_id);
  const float my_s = 1.0f / (1.0f + expf(-my_l));
  int id = 0;
  float s = 0.f, sum = 0.f;
  for (int r = 0; r < K; ++r) {
    const unsigned who = __ballot_sync(0xFFFFFFFFu, lane < K && rank == r);
    const int src = __ffs(who) - 1;
    const int id_r = __shfl_sync(0xFFFFFFFFu, my_id, src);
    const float s_r = __shfl_sync(0xFFFFFFFFu, my_s, src);
    sum += s_r;                    // slot order
    if (lane == r) {
      id = id_r;
      s = s_r;
    }
  }
  const float denom = fmaxf(sum, floor_);
  if (lane < K) {
    if ((flags & 1u) && (id < 0 || id >= E)) atomicOr(err, kErrBadId);
    ids[t * K + lane] = id;
    wts[t * K + lane] = s / denom;
  }
}

// ---------------------------------------------------------------------------------------------
// Expert-major permutation of the (token, slot) pairs: one CTA per two experts.
// counts[e] = number of pairs routed to e; offsets = exclusive prefix (E+1 entries);
// position p in [offsets[e], offsets[e+1]) lists the pairs of expert e by ascending token:
// perm[p] = t*K+k and inv[t*K+k] = p. Every CTA reads all P = T*K expert ids (L2-resident):
// pass 1 counts the pairs routed below e (its offset) and to e; a block scan over the threads'
// contiguous shares gives each thread its first position; pass 2 writes the pairs of e in pair
// order (a token routes to e at most once, so pair order is token order). No atomics decide an
// order, so the result is deterministic. Invalid ids count as expert 0 (and are flagged).
constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermChunk = 16;                   // ids a thread holds in registers per round
constexpr int kPermExperts = 2;                  // experts per CTA

__device__ __forceinline__ int clamp_id(int v, int E) { return (v < 0 || v >= E) ? 0 : v; }

// Loads ids [i0, i0 + 16) as four 16-byte vectors (entries past P are not read); i0 is a multiple of 16.
__device__ __forceinline__ void load_ids16(int (&v)[kPermChunk], const int* ids, int i0, int P) {
  if (i0 + kPermChunk <= P) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int4 w = __ldg(reinterpret_cast<const int4*>(ids + i0) + q);
      v[4 * q] = w.x;
      v[4 * q + 1] = w.y;
      v[4 * q + 2] = w.z;
      v[4 * q + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kPermChunk; ++j) v[j] = (i0 + j < P) ? __ldg(ids + i0 + j) : 0;
  }
}

// Counts the first `nv` of the thread's ids that are below e and equal to e.
__device__ __forceinline__ void count_ids(const int (&v)[kPermChunk], int nv, int e, int E, int& lt, int& eq,
                                          bool& bad) {
#pragma unroll
  for (int j = 0; j < kPermChunk; ++j) {
    if (j >= nv) continue;
    bad |= v[j] < 0 || v[j] >= E;
    const int c = clamp_id(v[j], E);
    lt += c < e;
    eq += c == e;
  }
}

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const int* __restrict__ ids, int P, int E,
                                                               int* __restrict__ counts, int* __restrict__ offsets,
                                                               int* __restrict__ perm, int* __restrict__ inv,
                                                               unsigned flags, unsigned* __restrict__ err) {
  __shared__ int w_sum[kPermWarps], w_base[kPermWarps];
  __shared__ int s_total;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kRound = kPermThreads * kPermChunk;
  // warp-order exclusive scan of one value per thread over the CTA; returns the exclusive prefix and
  // leaves the CTA total in s_total
  auto block_scan = [&](int x) -> int {
    int incl = x;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, m);
      if (lane >= m) incl += o;
    }
    __syncthreads();                               // w_sum / s_total of a previous scan are consumed
    if (lane == 31) w_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int c = w_sum[lane];
      int s = c;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, s, m);
        if (lane >= m) s += o;
      }
      w_base[lane] = s - c;
      if (lane == 31) s_total = s;
    }
    __syncthreads();
    return w_base[warp] + incl - x;
  };
  // the CTA's experts share the ids it loads (all of them in registers when P fits one round)
  int v[kPermChunk];
  for (int e = blockIdx.x * kPermExperts; e < min(E, blockIdx.x * kPermExperts + kPermExperts); ++e) {
    // pass 1: pairs routed below e (the offset of e)
    int lt = 0, eq_unused = 0;
    bool bad = false;
    for (int r0 = 0; r0 < P; r0 += kRound) {
      const int i0 = r0 + kPermChunk * tid;
      if (P > kRound || e == blockIdx.x * kPermExperts) load_ids16(v, ids, i0, P);
      count_ids(v, min(max(P - i0, 0), kPermChunk), e, E, lt, eq_unused, bad);
    }
    if (bad && (flags & 1u) && e == 0) atomicOr(err, kErrBadId);
    block_scan(lt);
    const int off = s_total;
    // pass 2: the pairs of e in pair order at off, off + 1, ...
    int run = 0;
    for (int r0 = 0; r0 < P; r0 += kRound) {
      const int i0 = r0 + kPermChunk * tid;
      const int nv = min(max(P - i0, 0), kPermChunk);
      if (P > kRound) load_ids16(v, ids, i0, P);   // one round: the ids are still in registers
      int l2 = 0, eq = 0;
      bool b2 = false;
      count_ids(v, nv, e, E, l2, eq, b2);
      int pos = off + run + block_scan(eq);
      run += s_total;
#pragma unroll
      for (int j = 0; j < kPermChunk; ++j) {
        if (j < nv && clamp_id(v[j], E) == e) {
          perm[pos] = i0 + j;
          inv[i0 + j] = pos;
          ++pos;
        }
      }
    }
    if (tid == 0) {
      counts[e] = run;
      offsets[e] = off;
      if (e == E - 1) offsets[E] = off + run;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Routed-expert activation operand of the prefill path: fp16(Hn x) per 128-segment for the int4
// format (the codes store W*blockdiag(Hn): Aijuus/flint-w4exp, weights row) or fp16(x) for NVFP4,
// written once per slot of the token at its permuted row inv[t][k], so that the rows of one expert
// are contiguous. One warp per (token, segment). For int4 every 8-block is stored in the order
// 0,4,1,5,2,6,3,7 to match the fp16 pairs the int4 decoder produces.
__global__ void __launch_bounds__(256) xg_kernel(const uint16_t* __restrict__ x, int T, int K,
                                                 const int* __restrict__ inv, int rotate, __half* __restrict__ xg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 8 + warp;
  const int t = gw / (kH / kGroup), seg = gw % (kH / kGroup);
  if (t >= T) return;
  const uint16_t* src = x + static_cast<size_t>(t) * kH + seg * kGroup + 4 * lane;
  const uint2 raw = ld_nc_v2(src);
  float v[4] = {bf16lo_to_f32(raw.x), bf16hi_to_f32(raw.x), bf16lo_to_f32(raw.y), bf16hi_to_f32(raw.y)};
  if (rotate) fwht128_warp(v);
  for (int k = 0; k < K; ++k) {
    const int prow = inv[t * K + k];
    store_seg_half(xg + static_cast<size_t>(prow) * kH + seg * kGroup, v, rotate != 0);
  }
}

// ---------------------------------------------------------------------------------------------
// host launchers

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, int T, int E, float* logits,
                                 cudaStream_t s) {
  dim3 grid((E + 7) / 8, (T + 7) / 8);
  router_logits_kernel<<<grid, 256, 0, s>>>(x, wr, T, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int nsplit, float* logits_out, int T, int E, int K, float floor_, int* ids,
                        float* wts, unsigned flags, unsigned* err, cudaStream_t s) {
  if (nsplit == kRouterSplit)
    topk_kernel<kRouterSplit><<<(T + 7) / 8, 256, 0, s>>>(logits, logits_out, T, E, K, floor_, ids, wts, flags, err);
  else if (nsplit == 1)
    topk_kernel<1><<<(T + 7) / 8, 256, 0, s>>>(logits, logits_out, T, E, K, floor_, ids, wts, flags, err);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_permute(const int* ids, int T, int K, int E, int* counts, int* offsets, int* perm, int* inv,
                           unsigned flags, unsigned* err, cudaStream_t s) {
  permute_kernel<<<(E + kPermExperts - 1) / kPermExperts, kPermThreads, 0, s>>>(ids, T * K, E, counts, offsets, perm, inv,
                                                                                  flags, err);
  return cudaGetLastError();
}

cudaError_t launch_xg(const uint16_t* x, int T, int K, const int* inv, int rotate, __half* xg, cudaStream_t s) {
  const int warps = T * (kH / kGroup);
  xg_kernel<<<(warps + 7) / 8, 256, 0, s>>>(x, T, K, inv, rotate, xg);
  return cudaGetLastError();
}

}  // namespace flint
