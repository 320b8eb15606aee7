// Kernel launchers of the Flint MoE library (internal interface between the host API and the
// device code).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace flint {

// Launches kernel<<<grid, threads, smem, s>>>(args...); with pdl as a programmatic dependent of the
// previous kernel in the stream (the kernel then calls griddepcontrol.wait before it reads that
// kernel's output, and may start its prologue while that kernel finishes).
template <typename Kern, typename... Args>
cudaError_t launch_pdl_kernel(Kern kernel, int grid, int threads, int smem, bool pdl, cudaStream_t s, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- decode path (T <= kDecodeMaxT): one persistent kernel, launched cooperatively ----
constexpr int kDecodeMaxT = 8;
constexpr int kMaxActive = 64;                 // active experts of a decode forward (T * top_k <= 64)
// Words of the decode kernel in the workspace (zeroed at create): the grid barrier (arrival count,
// generation, abort word) and the arrival counters of the 128-segments of h (each reset to zero by
// its last arriver).
enum : int {
  kCntBar = 0,                                 // [3]: count, generation, abort
  kCntSeg = 32,                                // [kMaxActive][4] gate|up tiles finished per 128-segment of h
  kCntInts = kCntSeg + 4 * kMaxActive
};

struct DecodeParams {
  CUtensorMap tm_gu;              // gate|up codes as 32-bit words [E*2I][H/8], box 64 words x 8 rows
  CUtensorMap tm_gu_sc;           // NVFP4 gate|up block scales as words [E*2I][H/64], box 8 words x 8 rows
  CUtensorMap tm_sh_gu;           // shared gate|up rows as 32-bit words [2Is][H/2], box 256 words x 2 rows
  CUtensorMap tm_sh_dn;           // shared down rows as 32-bit words [H][Is/2], box 64 words x 16 rows
  int fmt, T, E, K;
  float floor_, routed_scale;
  const uint16_t* x;              // [T][H] bf16
  const uint16_t* wr;             // [E][H] bf16
  const uint8_t* gu_codes;
  const uint8_t* gu_scales;
  const float* gu_ts;
  const uint8_t* dn_codes;
  const uint8_t* dn_scales;
  const float* dn_ts;
  const uint8_t* sh_gu;
  const uint8_t* sh_dn;
  uint16_t* y;                    // [T][H] bf16
  float* logits;                  // [T][E]
  int* ids;                       // [T][K]
  float* wts;                     // [T][K]
  int* counts;                    // [E]
  int* offsets;                   // [E+1]
  int* perm;                      // [P]
  int* inv;                       // [T][K]
  int* active;                    // [E]
  int* n_active;
  int4* etab;                     // [kMaxActive][2]: {e, offset, count, tokens (4 bits each)}, {ts_g, ts_u, ts_d, 0}
  __half* xq;                     // [T][H] fp16 activation operand of gate|up (NVFP4; int4: kept for inspection)
  uint8_t* xq8;                   // int4: [T][2][H] 16-bit fixed-point limbs (high s8, low u8) of Hn x
  float* xsc;                     // int4: [T][H/128] value of one unit of the limbs' 16-bit integer, / 16
  float* h32;                     // [P][I] SwiGLU output
  __half* hq;                     // NVFP4: [P][I] fp16 activation operand of down
  uint8_t* hq8;                   // int4: [P][2][I] limbs of Hn h
  float* hsc;                     // int4: [P][I/128] unit of hq8, / 16
  uint16_t* hs_hi;                // [T][Is] shared-expert SwiGLU output, bf16 pair
  uint16_t* hs_lo;
  float* ys;                      // [T][H] shared-expert output
  unsigned* err;
  int* cnt;                       // [kCntInts]
  const int* slot_of;             // [E] weight slot of each expert (weights in cache slots), or null
  int n_wslots;                   // weight slots when slot_of is set
  int route_in;                   // 1: ids and wts hold the routing already (no router, no top-k)
};

// Launches the decode kernel on `s` (grid = n_sm CTAs, cooperative). The caller has checked with
// decode_check_residency that one CTA fits per SM, and that n_sm >= kH / 16.
cudaError_t launch_decode(const DecodeParams& p, int n_sm, cudaStream_t s);
// Sets the kernel's shared-memory attributes and reports how many of its CTAs fit on one SM.
cudaError_t decode_check_residency(int fmt, int* blocks_per_sm);

// ---- prefill path (T > kDecodeMaxT): tcgen05 grouped GEMMs ----
enum PfPhase : int { kPhaseGateUp = 0, kPhaseDown = 1, kPhaseRouter = 2 };
constexpr int kRouterSplit = 4;            // K slices of the prefill router (partial logits summed by top-k)

struct PrefillParams {
  CUtensorMap tm_codes;           // routed: codes as 32-bit words [rows][K/8], box 16 words x 128 rows, 64-byte swizzle
  CUtensorMap tm_act;             // routed: fp16 activation rows (xg or hq), box 64 x 16 rows, 128-byte swizzle
  CUtensorMap tm_a;               // dense phases: bf16 weights (shared expert, router), box 64 x 128 rows, 128-byte swizzle
  CUtensorMap tm_b;               // shared: bf16 activations (x, or hs_hi), box 64 x 128 rows, 128-byte swizzle
  CUtensorMap tm_b2;              // shared down: hs_lo
  int T, top_k, E;
  const int* slot_of;             // [E] weight slot of each expert (weights in cache slots), or null
  int n_wslots;                   // weight slots when slot_of is set
  float* logits;                  // router phase output: partial logits [kRouterSplit][T][E]
  const int* offsets;             // [E+1]
  const int* perm;                // [P]
  const void* scales;             // int4 bf16 / nvfp4 e4m3, layout of the codes
  const float* tscale;            // gate|up [E][2] or down [E]; may be null
  __half* hq;                     // routed gate|up output [P][I]
  __half* o;                      // routed down output [P][H]
  uint16_t* hs_hi;                // shared gate|up output [T][Is], bf16 pair
  uint16_t* hs_lo;
  float* ys;                      // shared down output [T][H]
  unsigned* err;
  const float* act_ts;            // W4A4: activation rows' tensor scales [P]
  float* h32;                     // W4A4 gate|up output h [P][I] (fp32)
  const uint8_t* w_atoms;         // W4A4: weight block scales as MMA atoms [rows / 128][K/64][512]
  const uint8_t* act_atoms;       // W4A4: activation block scales as MMA atoms [chunk][K/64][512]
};

// pdl: launched as a programmatic dependent of the previous kernel in the stream (the routed down
// kernel streams its weights while the gate|up kernel finishes; it waits for it before reading h).
cudaError_t launch_prefill_routed(const PrefillParams& p, int fmt, int phase, int n_sm, bool pdl, cudaStream_t s);
cudaError_t launch_prefill_shared(const PrefillParams& p, int phase, int n_sm, cudaStream_t s, bool pdl = false);

// W4A4 (NVFP4 weights and activations). tm_codes: weight codes as bytes [rows][K/2], box 128 x 128
// rows, 128-byte swizzle; tm_act: activation codes [P][K/2], box 128 x 16 rows, 128-byte swizzle.
cudaError_t launch_w4a4_routed(const PrefillParams& p, int phase, int n_sm, bool pdl, cudaStream_t s);
// Chunks (64 permuted rows of one expert) the activation atom arrays must hold for P rows.
size_t w4a4_chunk_capacity(size_t P, int E);
// Weight block scales [rows][K/16] -> MMA atoms [rows / 128][K/64][512 bytes] (rows % 128 == 0).
cudaError_t launch_pack_sf_atoms(const uint8_t* scales, int rows, int K, uint8_t* atoms, cudaStream_t s);
// x (bf16 [T][H]) -> NVFP4 codes [P][H/2], scales [P][H/16], tensor scales [P] and scale atoms
// [chunk][H/64][512], written to each token's permuted rows inv[t][k]; rowc[p] = the row's chunk *
// 64 + its row in the chunk
cudaError_t launch_act_quant_x(const uint16_t* x, int T, int K, int E, const int* ids, const int* inv,
                               const int* offsets, const int* chunk_base, uint8_t* codes, uint8_t* scales,
                               uint8_t* atoms, float* ts, int* rowc, cudaStream_t s, bool pdl = false);
// h (fp32 [P][I]) -> codes [P][I/2], scales [P][I/16], tensor scales [P], atoms [chunk][I/64][512]
cudaError_t launch_act_quant_h(const float* h, int P, const int* rowc, uint8_t* codes, uint8_t* scales, uint8_t* atoms,
                               float* ts, bool pdl, cudaStream_t s);

// Residual stream of a layer stack: x (f32 [T][H]) += y (bf16, when not null); then, when z is not
// null, z = bf16(rmsnorm(x)) with eps.
cudaError_t launch_residual_rmsnorm(float* x, const uint16_t* y, int T, float eps, uint16_t* z, cudaStream_t s);
cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* wr, int T, int E, float* logits, cudaStream_t s);
// logits: `nsplit` partial logit arrays [nsplit][T][E], summed in slice order; the sums are also
// written to logits_out [T][E] when it is not null.
cudaError_t launch_topk(const float* logits, int nsplit, float* logits_out, int T, int E, int K, float floor_, int* ids,
                        float* wts, unsigned flags, unsigned* err, cudaStream_t s, bool pdl = false);
// chunk_base (may be null): [E] the first 64-row chunk of each expert, chunks numbered over all experts
// in ascending order (an exclusive prefix of ceil(count / 64)); the W4A4 path addresses its
// activation scale atoms by chunk.
cudaError_t launch_permute(const int* ids, int T, int K, int E, int* counts, int* offsets, int* perm, int* inv,
                           int* chunk_base, unsigned flags, unsigned* err, cudaStream_t s, bool pdl = false);
cudaError_t launch_xg(const uint16_t* x, int T, int K, const int* inv, int rotate, __half* xg, cudaStream_t s,
                      bool pdl = false);

cudaError_t launch_prefill_combine(const __half* o, const float* ys, const float* w, const int* inv, int T, int K,
                                   float routed_scale, uint16_t* y, bool pdl, cudaStream_t s);

}  // namespace flint
