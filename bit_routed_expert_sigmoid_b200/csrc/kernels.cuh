// Kernel launchers of the Flint MoE library (internal interface between the host API and the
// device code).
#pragma once

#include "common.cuh"

namespace flint {

struct GemvRouted {
  const uint8_t* codes;       // gate|up [E][2I][H/2] or down [E][H][I/2]
  const void* scales;         // int4 bf16 / nvfp4 e4m3, layout of the codes
  const float* tscale;        // gate|up [E][2] or down [E]; may be null
  const int* active;          // ascending experts with tokens
  const int* n_active;
  const int* offsets;         // [E+1]
  const int* perm;            // [P]
  int top_k;
  const __half* xq;           // gate|up input [T][H]
  float* h_out;               // gate|up output [P][I]
  const float* h_in;          // down input [P][I]
  float* o_out;               // down output [P][H]
};

struct GemvShared {
  const uint8_t* w_gu;        // bf16 [2Is][H]
  const uint8_t* w_dn;        // bf16 [H][Is]
  const uint16_t* x;          // bf16 [T][H]
  int T;
  uint16_t* hs_hi;            // bf16 [T][Is]
  uint16_t* hs_lo;
  float* ys;                  // [T][H]
};

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, int T, int E, float* logits, cudaStream_t s);
cudaError_t launch_topk(const float* logits, int T, int E, int K, float floor_, int* ids, float* wts, unsigned flags,
                        unsigned* err, cudaStream_t s);
cudaError_t launch_permute(const int* ids, int T, int K, int E, int* counts, int* offsets, int* perm, int* inv,
                           int* active, int* n_active, unsigned flags, unsigned* err, cudaStream_t s);
cudaError_t launch_xq(const uint16_t* x, int T, int rotate, __half* xq, cudaStream_t s);

cudaError_t launch_gu_routed(const GemvRouted& a, int fmt, int groups, cudaStream_t s);
cudaError_t launch_dn_routed(const GemvRouted& a, int fmt, int groups, cudaStream_t s);
cudaError_t launch_gu_shared(const GemvShared& a, cudaStream_t s);
cudaError_t launch_dn_shared(const GemvShared& a, cudaStream_t s);
cudaError_t launch_combine(const float* o, const float* ys, const float* w, const int* inv, int T, int K,
                           float routed_scale, uint16_t* y, cudaStream_t s);

}  // namespace flint
