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
// Selection runs on order-preserving 32-bit keys so that each of the k rounds is two warp reductions
// (redux.sync): the largest key, then the lowest index holding it. -0 is keyed as +0 (the two compare
// equal as logits) and NaN as 0, below every number, so it is picked only when nothing else is left.
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;   // NaN
  if ((u << 1) == 0u) u = 0u;                          // -0 as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int NS>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   float* __restrict__ logits_out, int T, int E, int K,
                                                   float floor_, int* __restrict__ ids, float* __restrict__ wts,
                                                   unsigned flags, unsigned* __restrict__ err) {
  pdl_wait();                                      // the logits are the previous kernel's output
  pdl_trigger();
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
    v[j] = a;
  }
  if (logits_out) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < per) logits_out[static_cast<size_t>(t) * E + lane + 32 * j] = v[j];
  }
  uint32_t key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) key[j] = logit_key(v[j]);
  unsigned live = (1u << per) - 1u;                // bit j: element lane+32j not yet chosen
  // the picks are warp-uniform: every lane keeps all of them
  int pid[kMaxTopK];
  uint32_t pkey[kMaxTopK];
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    pid[k] = 0x7FFFFFFF;           // unused slots sort last
    pkey[k] = 0u;
    if (k < K) {
      uint32_t lk = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if ((live >> j) & 1u) lk = max(lk, key[j]);
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, lk);
      uint32_t li = 0xFFFFFFFFu;
#pragma unroll
      for (int j = 7; j >= 0; --j)
        if (((live >> j) & 1u) && key[j] == m) li = static_cast<uint32_t>(lane + 32 * j);
      const uint32_t bi = __reduce_min_sync(0xFFFFFFFFu, li);
      if (static_cast<int>(bi & 31u) == lane) live &= ~(1u << (bi >> 5));
      pid[k] = static_cast<int>(bi);
      pkey[k] = m;
    }
  }
  // slots by ascending expert id (odd-even transposition network; the ids are distinct)
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
#pragma unroll
    for (int i = r & 1; i + 1 < kMaxTopK; i += 2) {
      if (pid[i] > pid[i + 1]) {
        const int ti = pid[i];
        pid[i] = pid[i + 1];
        pid[i + 1] = ti;
        const uint32_t tk = pkey[i];
        pkey[i] = pkey[i + 1];
        pkey[i + 1] = tk;
      }
    }
  }
  float s[kMaxTopK];
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k) {
    s[k] = 1.0f / (1.0f + expf(-key_logit(pkey[k])));
    if (k < K) sum += s[k];        // slot order
  }
  const float denom = fmaxf(sum, floor_);
  int id = 0;
  float sk = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k)
    if (lane == k) {
      id = pid[k];
      sk = s[k];
    }
  if (lane < K) {
    if ((flags & 1u) && (id < 0 || id >= E)) atomicOr(err, kErrBadId);
    ids[t * K + lane] = id;
    wts[t * K + lane] = sk / denom;
  }
}

// ---------------------------------------------------------------------------------------------
// Expert-major permutation of the (token, slot) pairs, a counting sort that keeps pair order.
// counts[e] = number of pairs routed to e; offsets = exclusive prefix (E+1 entries);
// position p in [offsets[e], offsets[e+1]) lists the pairs of expert e by ascending token:
// perm[p] = t*K+k and inv[t*K+k] = p. CTA c owns the 1024 pairs [1024c, 1024c + 1024), one per
// thread. It counts, in shared memory, every expert over all P pairs and over the pairs before its
// range (the ids are L2-resident), which gives the first position of each expert in its range; a
// pair's place among the equal ids of its range is its rank in its warp (match.any) plus the
// counts of the warps before it. Counts do not depend on the order of the shared-memory atomics, so
// the result is deterministic. A token routes to e at most once, so pair order is token order.
// Invalid ids count as expert 0 (and are flagged).
constexpr int kPermThreads = 1024;               // = pairs per CTA
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermUnroll = 4;                   // 16-byte id loads in flight per thread

__device__ __forceinline__ int clamp_id(int v, int E) { return (v < 0 || v >= E) ? 0 : v; }

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const int* __restrict__ ids, int P, int E,
                                                               int* __restrict__ counts, int* __restrict__ offsets,
                                                               int* __restrict__ perm, int* __restrict__ inv,
                                                               int* __restrict__ chunk_base, unsigned flags,
                                                               unsigned* __restrict__ err) {
  __shared__ int h_total[kMaxE], h_before[kMaxE], first[kMaxE];
  pdl_wait();                                      // the ids are the previous kernel's output
  pdl_trigger();
  __shared__ int wcnt[kPermWarps * kMaxE];        // [warp][expert]: pairs of the expert in the warp
  __shared__ int scan_w[kMaxE / 32], scan_c[kMaxE / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * kPermThreads;
  const int i = c0 + tid;
  const int raw = i < P ? __ldg(ids + i) : 0;
  for (int q = tid; q < E; q += kPermThreads) {
    h_total[q] = 0;
    h_before[q] = 0;
  }
  for (int q = tid; q < kPermWarps * E; q += kPermThreads) wcnt[q] = 0;
  __syncthreads();
  // histograms of all pairs and of the pairs before this range (ids + 4j is 16-byte aligned)
  bool bad = false;
  for (int r0 = 0; r0 < P; r0 += 4 * kPermThreads * kPermUnroll) {
    int v[4 * kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      const int j0 = r0 + 4 * (tid + u * kPermThreads);
      if (j0 + 4 <= P) {
        const int4 w = __ldg(reinterpret_cast<const int4*>(ids + j0));
        v[4 * u] = w.x;
        v[4 * u + 1] = w.y;
        v[4 * u + 2] = w.z;
        v[4 * u + 3] = w.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) v[4 * u + q] = (j0 + q < P) ? __ldg(ids + j0 + q) : 0;
      }
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = r0 + 4 * (tid + u * kPermThreads) + q;
        if (j < P) {
          bad |= v[4 * u + q] < 0 || v[4 * u + q] >= E;
          const int e = clamp_id(v[4 * u + q], E);
          atomicAdd(&h_total[e], 1);
          if (j < c0) atomicAdd(&h_before[e], 1);
        }
      }
    }
  }
  if (bad && (flags & 1u) && blockIdx.x == 0) atomicOr(err, kErrBadId);
  // this thread's pair: its rank among the equal ids of its warp
  const int e = i < P ? clamp_id(raw, E) : -1;
  const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
  const int rank_w = __popc(peers & ((1u << lane) - 1u));
  if (i < P && rank_w == 0) wcnt[warp * E + e] = __popc(peers);
  __syncthreads();
  // offsets: exclusive scan of the totals over the experts; per expert, exclusive scan of the warp
  // counts over the warps
  int incl = 0, tot = 0, incl_c = 0, nch = 0;
  if (tid < kMaxE) {
    tot = tid < E ? h_total[tid] : 0;
    incl = tot;
    nch = (tot + 63) >> 6;                         // 64-row chunks of the expert (W4A4 chunk numbering)
    incl_c = nch;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, m), oc = __shfl_up_sync(0xFFFFFFFFu, incl_c, m);
      if (lane >= m) {
        incl += o;
        incl_c += oc;
      }
    }
    if (lane == 31) {
      scan_w[warp] = incl;
      scan_c[warp] = incl_c;
    }
    if (tid < E) {
      int c[kPermWarps];
#pragma unroll
      for (int w = 0; w < kPermWarps; ++w) c[w] = wcnt[w * E + tid];
      int run = 0;
#pragma unroll
      for (int w = 0; w < kPermWarps; ++w) {
        wcnt[w * E + tid] = run;
        run += c[w];
      }
    }
  }
  __syncthreads();
  if (tid < E) {
    int off = incl - tot;
    for (int w = 0; w < warp; ++w) off += scan_w[w];
    first[tid] = off + h_before[tid];
    if (blockIdx.x == 0) {
      counts[tid] = tot;
      offsets[tid] = off;
      if (tid == E - 1) offsets[E] = off + tot;
      if (chunk_base) {
        int cb = incl_c - nch;
        for (int w = 0; w < warp; ++w) cb += scan_c[w];
        chunk_base[tid] = cb;
      }
    }
  }
  __syncthreads();
  if (i < P) {
    const int pos = first[e] + wcnt[warp * E + e] + rank_w;
    perm[pos] = i;
    inv[i] = pos;
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
  pdl_wait();                                      // inv is the previous kernel's output
  pdl_trigger();
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
                        float* wts, unsigned flags, unsigned* err, cudaStream_t s, bool pdl) {
  if (nsplit == kRouterSplit)
    return launch_pdl_kernel(topk_kernel<kRouterSplit>, (T + 7) / 8, 256, 0, pdl, s, logits, logits_out, T, E, K,
                             floor_, ids, wts, flags, err);
  if (nsplit == 1)
    return launch_pdl_kernel(topk_kernel<1>, (T + 7) / 8, 256, 0, pdl, s, logits, logits_out, T, E, K, floor_, ids,
                             wts, flags, err);
  return cudaErrorInvalidValue;
}

cudaError_t launch_permute(const int* ids, int T, int K, int E, int* counts, int* offsets, int* perm, int* inv,
                           int* chunk_base, unsigned flags, unsigned* err, cudaStream_t s, bool pdl) {
  const int P = T * K;
  const int grid = P > 0 ? (P + kPermThreads - 1) / kPermThreads : 1;
  return launch_pdl_kernel(permute_kernel, grid, kPermThreads, 0, pdl, s, ids, P, E, counts, offsets, perm, inv, chunk_base,
                           flags, err);
}

cudaError_t launch_xg(const uint16_t* x, int T, int K, const int* inv, int rotate, __half* xg, cudaStream_t s,
                      bool pdl) {
  const int warps = T * (kH / kGroup);
  return launch_pdl_kernel(xg_kernel, (warps + 7) / 8, 256, 0, pdl, s, x, T, K, inv, rotate, xg);
}

}  // namespace flint
