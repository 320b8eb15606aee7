// Routing stage of the Flint MoE layer: router logits, unbiased sigmoid top-k with the
// selected-sum floor, the expert-major permutation of (token, slot) pairs, and the activation
// operand of the routed experts (x rotated per 128-segment for the int4 format).
#include "kernels.cuh"

namespace flint {

// ---------------------------------------------------------------------------------------------
// Router logits on CUDA cores: logits[t][e] = sum_j W_r[e][j] * x[t][j]. The bf16 x bf16 products
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
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                   float floor_, int* __restrict__ ids, float* __restrict__ wts,
                                                   unsigned flags, unsigned* __restrict__ err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const int per = E >> 5;          // logits per lane (E is a multiple of 32, at most 256)
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = (j < per) ? logits[static_cast<size_t>(t) * E + lane + 32 * j] : -INFINITY;
  unsigned taken = 0;              // bit j: element lane+32j already chosen
  int chosen[kMaxTopK];
  float chosen_l[kMaxTopK];
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
    chosen[k] = bi;
    chosen_l[k] = bv;
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
  }
  // order the slots by expert id; lane k < K writes slot k
  float s_sorted[kMaxTopK];
  int id_sorted[kMaxTopK];
  for (int k = 0; k < K; ++k) {
    int rank = 0;
    for (int j = 0; j < K; ++j) rank += (chosen[j] < chosen[k]);
    id_sorted[rank] = chosen[k];
    s_sorted[rank] = 1.0f / (1.0f + expf(-chosen_l[k]));
  }
  float sum = 0.f;
  for (int k = 0; k < K; ++k) sum += s_sorted[k];
  const float denom = fmaxf(sum, floor_);
  if (lane < K) {
    int id = 0;
    float s = 0.f;
    for (int k = 0; k < K; ++k)
      if (k == lane) { id = id_sorted[k]; s = s_sorted[k]; }
    if ((flags & 1u) && (id < 0 || id >= E)) atomicOr(err, kErrBadId);
    ids[t * K + lane] = id;
    wts[t * K + lane] = s / denom;
  }
}

// ---------------------------------------------------------------------------------------------
// Expert-major permutation of the (token, slot) pairs, one CTA of 512 threads.
// counts[e] = number of pairs routed to e; offsets = exclusive prefix (E+1 entries);
// position p in [offsets[e], offsets[e+1]) lists the pairs of expert e by ascending token:
// perm[p] = t*K+k and inv[t*K+k] = p. Ranks come from per-warp bitmasks and prefix sums, never
// from the order atomics happen to run in, so the result is deterministic. Also lists the experts
// that received tokens (ascending) in active[0..n_active).
constexpr int kPermThreads = 512;
constexpr int kPermWarps = kPermThreads / 32;

__global__ void __launch_bounds__(kPermThreads) permute_kernel(const int* __restrict__ ids, int T, int K, int E,
                                                               int* __restrict__ counts, int* __restrict__ offsets,
                                                               int* __restrict__ perm, int* __restrict__ inv,
                                                               int* __restrict__ active, int* __restrict__ n_active,
                                                               unsigned flags, unsigned* __restrict__ err) {
  __shared__ int cnt[kMaxE];
  __shared__ int run[kMaxE];
  __shared__ unsigned mask[kPermWarps][kMaxE];
  __shared__ int base[kPermWarps][kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < kMaxE; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  const int P = T * K;
  for (int i = tid; i < P; i += kPermThreads) {
    int e = ids[i];
    if (e < 0 || e >= E) {
      if (flags & 1u) atomicOr(err, kErrBadId);
      e = 0;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // exclusive scan over experts by warp 0 (8 experts per lane)
  if (warp == 0) {
    int loc[8];
    int s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      loc[j] = s;
      s += (e < E) ? cnt[e] : 0;
    }
    int incl = s;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, m);
      if (lane >= m) incl += o;
    }
    const int excl = incl - s;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) {
        offsets[e] = excl + loc[j];
        run[e] = excl + loc[j];
        counts[e] = cnt[e];
      }
    }
    if (lane == 31) offsets[E] = incl;
    // active experts (count > 0), ascending
    int fl[8];
    int fs = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      fl[j] = fs;
      fs += (e < E && cnt[e] > 0) ? 1 : 0;
    }
    int finc = fs;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, finc, m);
      if (lane >= m) finc += o;
    }
    const int fex = finc - fs;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E && cnt[e] > 0) active[fex + fl[j]] = e;
    }
    if (lane == 31) *n_active = finc;
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int t0 = 0; t0 < T; t0 += kPermThreads) {
    for (int e = lane; e < kMaxE; e += 32) mask[warp][e] = 0u;
    __syncwarp();
    const int t = t0 + tid;
    int my_e[kMaxTopK];
    if (t < T) {
      for (int k = 0; k < K; ++k) {
        int e = ids[t * K + k];
        if (e < 0 || e >= E) e = 0;
        my_e[k] = e;
        atomicOr(&mask[warp][e], 1u << lane);
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads) {
      int b = run[e];
      for (int w = 0; w < kPermWarps; ++w) {
        base[w][e] = b;
        b += __popc(mask[w][e]);
      }
      run[e] = b;
    }
    __syncthreads();
    if (t < T) {
      for (int k = 0; k < K; ++k) {
        const int e = my_e[k];
        const int p = base[warp][e] + __popc(mask[warp][e] & lt_mask);
        perm[p] = t * K + k;
        inv[t * K + k] = p;
      }
    }
    __syncthreads();
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

cudaError_t launch_topk(const float* logits, int T, int E, int K, float floor_, int* ids, float* wts, unsigned flags,
                        unsigned* err, cudaStream_t s) {
  topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, K, floor_, ids, wts, flags, err);
  return cudaGetLastError();
}

cudaError_t launch_permute(const int* ids, int T, int K, int E, int* counts, int* offsets, int* perm, int* inv,
                           int* active, int* n_active, unsigned flags, unsigned* err, cudaStream_t s) {
  permute_kernel<<<1, kPermThreads, 0, s>>>(ids, T, K, E, counts, offsets, perm, inv, active, n_active, flags, err);
  return cudaGetLastError();
}

cudaError_t launch_xg(const uint16_t* x, int T, int K, const int* inv, int rotate, __half* xg, cudaStream_t s) {
  const int warps = T * (kH / kGroup);
  xg_kernel<<<(warps + 7) / 8, 256, 0, s>>>(x, T, K, inv, rotate, xg);
  return cudaGetLastError();
}

}  // namespace flint
