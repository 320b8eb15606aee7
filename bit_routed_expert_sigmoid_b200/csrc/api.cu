// Host side of the Flint MoE C ABI: argument checks, workspace plan and the launch sequence.
// The library allocates no device memory: weights, activations and workspace belong to the caller.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/flint_moe.h"
#include "kernels.cuh"

using namespace flint;

struct flint_moe_ctx {
  flint_moe_cfg cfg;
  flint_moe_weights w;
  char* ws;
  size_t ws_bytes;
  // workspace carve-up
  float* logits;
  float* logits_part;
  int* ids;
  float* wts;
  int* counts;
  int* offsets;
  int* perm;
  int* inv;
  int* active;
  int* n_active;
  int* slot_of;                            // [kMaxE] weight slot of each expert (cache mode)
  int4* etab;
  int* cnt;
  unsigned* err;
  __half* xq;
  __half* xg;
  uint8_t* xq8;
  float* xsc;
  float* h32;
  __half* hq;
  uint8_t* hq8;
  float* hsc;
  uint16_t* hs_hi;
  uint16_t* hs_lo;
  float* o;
  float* ys;
  uint16_t* x_stage;
  uint16_t* y_stage;
  uint8_t* xa;                             // W4A4: x codes [P][H/2], scales [P][H/16], tensor scales [P]
  uint8_t* xa_sf;
  float* xa_ts;
  uint8_t* ha;                             // W4A4: h codes [P][I/2], scales [P][I/16], tensor scales [P]
  uint8_t* ha_sf;
  float* ha_ts;
  int* rowc;                               // W4A4: chunk position (chunk * 64 + row in chunk) of each permuted row
  int* chunk_base;                         // W4A4: [E] first 64-row chunk of each expert
  uint8_t* xa_atoms;                       // W4A4: block scales of x and h as MMA atoms [chunk][K/64][512]
  uint8_t* ha_atoms;
  uint8_t* w_atoms_gu;                     // W4A4: weight block scales as MMA atoms [rows / 128][K/64][512]
  uint8_t* w_atoms_dn;
  int last_T;
  bool w4a4;
  int n_sm;
  CUtensorMap tm_gu, tm_gu_sc, tm_sh_gu, tm_sh_dn;  // tensor maps of the decode kernel's weight copies
  CUtensorMap tm_pf_gu, tm_pf_dn;          // prefill: routed codes, 16-word x 128-row boxes, 64-byte swizzle
  CUtensorMap tm_pf_sh_gu, tm_pf_sh_dn;    // prefill: shared-expert weights, 64 x 128 bf16 boxes
  CUtensorMap tm_pf_router;                // prefill: router rows [E][H], 64 x 128 bf16 boxes
  CUtensorMap tm_pf_hs_hi, tm_pf_hs_lo;    // prefill: shared-expert hidden pair [t_max][Is]
  CUtensorMap tm_pf_xg, tm_pf_hq;          // prefill: routed activation rows (fp16, 64 x 16 boxes)
  CUtensorMap tm_w4_gu, tm_w4_dn;          // W4A4: weight codes as bytes, 128 x 128-row boxes, 128-byte swizzle
  CUtensorMap tm_w4_xa, tm_w4_ha;          // W4A4: activation codes, 128 x 16-row boxes, 128-byte swizzle
  // instrumentation (caller-owned cudaEvent_t handles)
  cudaEvent_t events[32];
  int n_events;
  // prefill: the routing chain runs on `side` (higher priority) while the shared expert runs on the
  // caller's stream; ev_fork / ev_join order the two
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
  ~flint_moe_ctx() {
    if (ev_join) cudaEventDestroy(ev_join);
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (side) cudaStreamDestroy(side);
  }
};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

flint_status check_cfg(const flint_moe_cfg* c) {
  if (!c) return FLINT_ERR_INVALID_ARG;
  if (c->t_max < 1 || c->t_max > 16384) return FLINT_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > kMaxTopK) return FLINT_ERR_INVALID_ARG;
  if (c->n_experts < c->top_k || c->n_experts <= 0) return FLINT_ERR_INVALID_ARG;
  if (c->fmt != FLINT_W_INT4_G128_FWHT128 && c->fmt != FLINT_W_NVFP4) return FLINT_ERR_INVALID_ARG;
  if (!(c->norm_floor > 0.f) || !(c->routed_scale == c->routed_scale)) return FLINT_ERR_INVALID_ARG;
  if (c->hidden != kH || c->inter != kI || c->inter_shared != kIs) return FLINT_ERR_UNSUPPORTED;
  if (c->n_experts % 32 != 0 || c->n_experts > kMaxE) return FLINT_ERR_UNSUPPORTED;
  if (c->n_slots < 0 || c->n_slots > c->n_experts) return FLINT_ERR_INVALID_ARG;
  if ((c->flags & FLINT_FLAG_W4A4) && (c->fmt != FLINT_W_NVFP4 || c->n_slots > 0)) return FLINT_ERR_UNSUPPORTED;
  return FLINT_OK;
}

// cuTensorMapEncodeTiled, from the driver through the runtime (no link-time driver dependency).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D map of `rows` rows of `row_bytes` bytes viewed as 32-bit words; box of box_words x box_rows.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_words,
                 uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes / 4, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_words, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over `rows` rows of `row_bytes` bytes with elements of `dtype` (`elem` bytes each); box of
// box_inner elements x box_rows rows, with the given swizzle. Rows past `rows` read as zeros.
bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, uint32_t elem, uint64_t rows,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes / elem, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16_tiles(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_f16_rows16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, rows, cols * 2, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
}

// W4A4 codes: bytes, box of 128 bytes x box_rows rows with the 128-byte swizzle
bool encode_fp4_tiles(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  return encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, row_bytes, 128, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_code_tiles(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes) {
  return encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, rows, row_bytes, 16, 128, CU_TENSOR_MAP_SWIZZLE_64B);
}

// Side stream of the prefill routing chain, at the highest priority (it is the longer branch).
bool create_side_stream(flint_moe_ctx* h) {
  int lo = 0, hi = 0;
  if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return false;
  return cudaStreamCreateWithPriority(&h->side, cudaStreamNonBlocking, hi) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) == cudaSuccess;
}

// Lays the workspace out; with base == nullptr only the size is computed.
size_t plan(flint_moe_ctx* h, const flint_moe_cfg& c, char* base) {
  const size_t T = c.t_max, E = c.n_experts, K = c.top_k, P = T * K;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  char* p_logits = take(T * E * 4);
  char* p_lpart = take(kRouterSplit * T * E * 4);
  char* p_ids = take(P * 4);
  char* p_wts = take(P * 4);
  char* p_counts = take(E * 4);
  char* p_offsets = take((E + 1) * 4);
  char* p_perm = take(P * 4);
  char* p_inv = take(P * 4);
  char* p_active = take(E * 4);
  char* p_nact = take(16);
  char* p_slot = take(kMaxE * 4);
  char* p_etab = take(kMaxActive * 2 * 16);
  char* p_cnt = take(kCntInts * 4);
  char* p_err = take(16);
  char* p_xq = take(T * kH * 2);
  char* p_xg = take(P * kH * 2);
  char* p_xq8 = take(T * kH * 2);
  char* p_xsc = take(T * (kH / kGroup) * 4);
  char* p_h32 = take(P * kI * 4);
  char* p_hq = take(P * kI * 2);
  char* p_hq8 = take(P * kI * 2);
  char* p_hsc = take(P * (kI / kGroup) * 4);
  char* p_hs_hi = take(T * kIs * 2);
  char* p_hs_lo = take(T * kIs * 2);
  char* p_o = take(P * kH * 4);
  char* p_ys = take(T * kH * 4);
  char* p_xs = take(T * kH * 2);
  char* p_ys2 = take(T * kH * 2);
  const size_t PA = (c.flags & FLINT_FLAG_W4A4) ? P : 0;      // W4A4 buffers only when asked for
  char* p_xa = take(PA * kH / 2);
  char* p_xa_sf = take(PA * kH / 16);
  char* p_xa_ts = take(PA * 4);
  char* p_ha = take(PA * kI / 2);
  char* p_ha_sf = take(PA * kI / 16);
  char* p_ha_ts = take(PA * 4);
  const size_t CA = PA ? w4a4_chunk_capacity(P, static_cast<int>(E)) : 0;
  const size_t WR = PA ? static_cast<size_t>(c.n_experts) : 0;          // W4A4 handles take no cache slots
  char* p_rowc = take(PA * 4);
  char* p_cbase = take(PA ? E * 4 : 0);
  char* p_xa_atoms = take(CA * (kH / 64) * 512);
  char* p_ha_atoms = take(CA * (kI / 64) * 512);
  char* p_w_atoms_gu = take(WR * (2 * kI / 128) * (kH / 64) * 512);
  char* p_w_atoms_dn = take(WR * (kH / 128) * (kI / 64) * 512);
  if (h) {
    h->logits = reinterpret_cast<float*>(p_logits);
    h->logits_part = reinterpret_cast<float*>(p_lpart);
    h->ids = reinterpret_cast<int*>(p_ids);
    h->wts = reinterpret_cast<float*>(p_wts);
    h->counts = reinterpret_cast<int*>(p_counts);
    h->offsets = reinterpret_cast<int*>(p_offsets);
    h->perm = reinterpret_cast<int*>(p_perm);
    h->inv = reinterpret_cast<int*>(p_inv);
    h->active = reinterpret_cast<int*>(p_active);
    h->n_active = reinterpret_cast<int*>(p_nact);
    h->slot_of = reinterpret_cast<int*>(p_slot);
    h->etab = reinterpret_cast<int4*>(p_etab);
    h->cnt = reinterpret_cast<int*>(p_cnt);
    h->err = reinterpret_cast<unsigned*>(p_err);
    h->xq = reinterpret_cast<__half*>(p_xq);
    h->xg = reinterpret_cast<__half*>(p_xg);
    h->h32 = reinterpret_cast<float*>(p_h32);
    h->hq = reinterpret_cast<__half*>(p_hq);
    h->xq8 = reinterpret_cast<uint8_t*>(p_xq8);
    h->xsc = reinterpret_cast<float*>(p_xsc);
    h->hq8 = reinterpret_cast<uint8_t*>(p_hq8);
    h->hsc = reinterpret_cast<float*>(p_hsc);
    h->hs_hi = reinterpret_cast<uint16_t*>(p_hs_hi);
    h->hs_lo = reinterpret_cast<uint16_t*>(p_hs_lo);
    h->o = reinterpret_cast<float*>(p_o);
    h->ys = reinterpret_cast<float*>(p_ys);
    h->x_stage = reinterpret_cast<uint16_t*>(p_xs);
    h->y_stage = reinterpret_cast<uint16_t*>(p_ys2);
    h->xa = reinterpret_cast<uint8_t*>(p_xa);
    h->xa_sf = reinterpret_cast<uint8_t*>(p_xa_sf);
    h->xa_ts = reinterpret_cast<float*>(p_xa_ts);
    h->ha = reinterpret_cast<uint8_t*>(p_ha);
    h->ha_sf = reinterpret_cast<uint8_t*>(p_ha_sf);
    h->ha_ts = reinterpret_cast<float*>(p_ha_ts);
    h->rowc = reinterpret_cast<int*>(p_rowc);
    h->chunk_base = reinterpret_cast<int*>(p_cbase);
    h->xa_atoms = reinterpret_cast<uint8_t*>(p_xa_atoms);
    h->ha_atoms = reinterpret_cast<uint8_t*>(p_ha_atoms);
    h->w_atoms_gu = reinterpret_cast<uint8_t*>(p_w_atoms_gu);
    h->w_atoms_dn = reinterpret_cast<uint8_t*>(p_w_atoms_dn);
  }
  return off;
}

// T <= kDecodeMaxT: one kernel; larger T: one kernel per step.
const char* const kDecodeStages[] = {"layer"};
const char* const kGemvStages[] = {"router_logits", "topk", "permute", "xq", "gu_shared",
                                   "gu_routed", "dn_routed", "dn_shared", "combine"};
// W4A4: the SwiGLU output is quantised between the routed projections
const char* const kW4a4Stages[] = {"router_logits", "topk", "permute", "xq", "gu_shared",
                                   "gu_routed", "hq", "dn_routed", "dn_shared", "combine"};

template <size_t N>
constexpr int count_of(const char* const (&)[N]) {
  return static_cast<int>(N);
}

int stage_count(const flint_moe_ctx* h, int T) {
  if (T <= kDecodeMaxT) return count_of(kDecodeStages);
  return h->w4a4 ? count_of(kW4a4Stages) : count_of(kGemvStages);
}

const char* stage_name(const flint_moe_ctx* h, int T, int i) {
  if (i < 0 || i >= stage_count(h, T)) return nullptr;
  if (T <= kDecodeMaxT) return kDecodeStages[i];
  return h->w4a4 ? kW4a4Stages[i] : kGemvStages[i];
}

// Records the next instrumentation event, if any.
struct StageMarks {
  flint_moe_ctx* h;
  cudaStream_t s;
  int next;
  cudaError_t mark() {
    if (h->n_events == 0 || next >= h->n_events) return cudaSuccess;
    return cudaEventRecord(h->events[next++], s);
  }
};

#define FLINT_TRY(expr)                        \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return FLINT_ERR_CUDA; \
  } while (0)

// route_in: h->ids and h->wts already hold this forward's routing (no router, no top-k).
flint_status run_forward(flint_moe_ctx* h, const uint16_t* x, int T, uint16_t* y, cudaStream_t s, bool route_in = false) {
  const flint_moe_cfg& c = h->cfg;
  const int E = c.n_experts, K = c.top_k;
  const int fmt = c.fmt == FLINT_W_INT4_G128_FWHT128 ? kInt4 : kNvfp4;
  StageMarks m{h, s, 0};
  FLINT_TRY(m.mark());
  if (T <= kDecodeMaxT) {
    DecodeParams d{};
    d.tm_gu = h->tm_gu;
    d.tm_gu_sc = h->tm_gu_sc;
    d.tm_sh_gu = h->tm_sh_gu;
    d.tm_sh_dn = h->tm_sh_dn;
    d.fmt = fmt;
    d.T = T;
    d.E = E;
    d.K = K;
    d.floor_ = c.norm_floor;
    d.routed_scale = c.routed_scale;
    d.x = x;
    d.wr = static_cast<const uint16_t*>(h->w.router_w);
    d.gu_codes = static_cast<const uint8_t*>(h->w.gu_codes);
    d.gu_scales = static_cast<const uint8_t*>(h->w.gu_scales);
    d.gu_ts = h->w.gu_tscale;
    d.dn_codes = static_cast<const uint8_t*>(h->w.dn_codes);
    d.dn_scales = static_cast<const uint8_t*>(h->w.dn_scales);
    d.dn_ts = h->w.dn_tscale;
    d.sh_gu = static_cast<const uint8_t*>(h->w.sh_gu);
    d.sh_dn = static_cast<const uint8_t*>(h->w.sh_dn);
    d.y = y;
    d.logits = h->logits;
    d.ids = h->ids;
    d.wts = h->wts;
    d.counts = h->counts;
    d.offsets = h->offsets;
    d.perm = h->perm;
    d.inv = h->inv;
    d.active = h->active;
    d.n_active = h->n_active;
    d.etab = h->etab;
    d.xq = h->xq;
    d.h32 = h->h32;
    d.hq = h->hq;
    d.xq8 = h->xq8;
    d.xsc = h->xsc;
    d.hq8 = h->hq8;
    d.hsc = h->hsc;
    d.hs_hi = h->hs_hi;
    d.hs_lo = h->hs_lo;
    d.ys = h->ys;
    d.err = h->err;
    d.cnt = h->cnt;
    d.slot_of = c.n_slots > 0 ? h->slot_of : nullptr;
    d.n_wslots = c.n_slots;
    d.route_in = route_in ? 1 : 0;
    FLINT_TRY(launch_decode(d, h->n_sm, s));
    FLINT_TRY(m.mark());
    return FLINT_OK;
  }
  PrefillParams pp{};
  pp.T = T;
  pp.top_k = K;
  pp.E = E;
  pp.logits = h->logits_part;
  pp.offsets = h->offsets;
  pp.perm = h->perm;
  pp.hq = h->hq;
  pp.o = reinterpret_cast<__half*>(h->o);          // fp16 [P][H] view of the fp32 buffer
  pp.hs_hi = h->hs_hi;
  pp.hs_lo = h->hs_lo;
  pp.ys = h->ys;
  pp.err = h->err;
  pp.slot_of = c.n_slots > 0 ? h->slot_of : nullptr;
  pp.n_wslots = c.n_slots;
  // B = x as given (map encoded per call: x changes, rows past T read as zeros)
  CUtensorMap tm_x;
  if (!encode_bf16_tiles(&tm_x, x, T, kH)) return FLINT_ERR_CUDA;
  // The routing chain (router, top-k, permutation, activation operand) and the shared expert are
  // independent; without instrumentation the chain runs on the side stream while the shared
  // expert's kernels (which leave SMs free) run on `s`. With instrumentation everything runs on `s`
  // in stage order.
  const bool fork = h->n_events == 0 && h->side != nullptr;
  // routed down and combine start as programmatic dependents of their predecessor (not between
  // instrumentation events, which serialise the stages anyway)
  const bool pdl = h->n_events == 0;
  cudaStream_t rs = fork ? h->side : s;
  if (fork) {
    FLINT_TRY(cudaEventRecord(h->ev_fork, s));
    FLINT_TRY(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
  }
  if (!route_in) {
    pp.tm_a = h->tm_pf_router;
    pp.tm_b = tm_x;
    FLINT_TRY(launch_prefill_shared(pp, kPhaseRouter, h->n_sm, rs));
    FLINT_TRY(m.mark());
    FLINT_TRY(launch_topk(h->logits_part, kRouterSplit, h->logits, T, E, K, c.norm_floor, h->ids, h->wts, c.flags, h->err, rs,
                          pdl));
    FLINT_TRY(m.mark());
  }
  // the chain's kernels are programmatic dependents of their predecessor (the permutation only when the
  // top-k ran right before it on this stream)
  FLINT_TRY(launch_permute(h->ids, T, K, E, h->counts, h->offsets, h->perm, h->inv, h->w4a4 ? h->chunk_base : nullptr,
                           c.flags, h->err, rs, pdl && !route_in));
  FLINT_TRY(m.mark());
  if (h->w4a4)
    FLINT_TRY(launch_act_quant_x(x, T, K, E, h->ids, h->inv, h->offsets, h->chunk_base, h->xa, h->xa_sf, h->xa_atoms,
                                 h->xa_ts, h->rowc, rs, pdl));
  else FLINT_TRY(launch_xg(x, T, K, h->inv, fmt == kInt4 ? 1 : 0, h->xg, rs, pdl));
  FLINT_TRY(m.mark());

  pp.tm_a = h->tm_pf_sh_gu;                        // shared gate|up: B = x
  pp.tm_b = tm_x;
  FLINT_TRY(launch_prefill_shared(pp, kPhaseGateUp, h->n_sm, s));
  FLINT_TRY(m.mark());
  if (fork) {                                      // shared down right behind shared gate|up
    pp.tm_a = h->tm_pf_sh_dn;
    pp.tm_b = h->tm_pf_hs_hi;
    pp.tm_b2 = h->tm_pf_hs_lo;
    FLINT_TRY(launch_prefill_shared(pp, kPhaseDown, h->n_sm, s, pdl));
    FLINT_TRY(cudaEventRecord(h->ev_join, h->side));
    FLINT_TRY(cudaStreamWaitEvent(s, h->ev_join, 0));
  }
  if (h->w4a4) {
    pp.tm_codes = h->tm_w4_gu;
    pp.w_atoms = h->w_atoms_gu;
    pp.tm_act = h->tm_w4_xa;
    pp.act_atoms = h->xa_atoms;
    pp.act_ts = h->xa_ts;
    pp.tscale = h->w.gu_tscale;
    pp.h32 = h->h32;
    FLINT_TRY(launch_w4a4_routed(pp, kPhaseGateUp, h->n_sm, false, s));
    FLINT_TRY(m.mark());
    FLINT_TRY(launch_act_quant_h(h->h32, T * K, h->rowc, h->ha, h->ha_sf, h->ha_atoms, h->ha_ts, pdl, s));
    FLINT_TRY(m.mark());
    pp.tm_codes = h->tm_w4_dn;
    pp.w_atoms = h->w_atoms_dn;
    pp.tm_act = h->tm_w4_ha;
    pp.act_atoms = h->ha_atoms;
    pp.act_ts = h->ha_ts;
    pp.tscale = h->w.dn_tscale;
    FLINT_TRY(launch_w4a4_routed(pp, kPhaseDown, h->n_sm, pdl, s));
    FLINT_TRY(m.mark());
  } else {
    pp.tm_codes = h->tm_pf_gu;
    pp.tm_act = h->tm_pf_xg;
    pp.scales = h->w.gu_scales;
    pp.tscale = h->w.gu_tscale;
    FLINT_TRY(launch_prefill_routed(pp, fmt, kPhaseGateUp, h->n_sm, false, s));
    FLINT_TRY(m.mark());
    pp.tm_codes = h->tm_pf_dn;
    pp.tm_act = h->tm_pf_hq;
    pp.scales = h->w.dn_scales;
    pp.tscale = h->w.dn_tscale;
    FLINT_TRY(launch_prefill_routed(pp, fmt, kPhaseDown, h->n_sm, pdl, s));
    FLINT_TRY(m.mark());
  }
  if (!fork) {
    pp.tm_a = h->tm_pf_sh_dn;
    pp.tm_b = h->tm_pf_hs_hi;
    pp.tm_b2 = h->tm_pf_hs_lo;
    FLINT_TRY(launch_prefill_shared(pp, kPhaseDown, h->n_sm, s));
    FLINT_TRY(m.mark());
  }
  FLINT_TRY(launch_prefill_combine(reinterpret_cast<const __half*>(h->o), h->ys, h->wts, h->inv, T, K, c.routed_scale, y, pdl, s));
  FLINT_TRY(m.mark());
  return FLINT_OK;
}

}  // namespace

extern "C" {

size_t flint_moe_workspace_size(const flint_moe_cfg* cfg) {
  if (check_cfg(cfg) != FLINT_OK) return 0;
  return plan(nullptr, *cfg, nullptr);
}

flint_status flint_moe_create(const flint_moe_cfg* cfg, const flint_moe_weights* weights, void* workspace,
                              size_t workspace_bytes, flint_moe_t* out) {
  if (!out) return FLINT_ERR_INVALID_ARG;
  *out = nullptr;
  flint_status st = check_cfg(cfg);
  if (st != FLINT_OK) return st;
  if (!weights) return FLINT_ERR_INVALID_ARG;
  const flint_moe_weights& w = *weights;
  if (!aligned16(w.router_w) || !aligned16(w.gu_codes) || !aligned16(w.gu_scales) || !aligned16(w.dn_codes) ||
      !aligned16(w.dn_scales) || !aligned16(w.sh_gu) || !aligned16(w.sh_dn))
    return FLINT_ERR_INVALID_ARG;
  if (cfg->fmt == FLINT_W_NVFP4 && (!w.gu_tscale || !w.dn_tscale)) return FLINT_ERR_INVALID_ARG;
  if ((w.gu_tscale && (reinterpret_cast<uintptr_t>(w.gu_tscale) & 7u)) ||
      (w.dn_tscale && (reinterpret_cast<uintptr_t>(w.dn_tscale) & 3u)))
    return FLINT_ERR_INVALID_ARG;
  const size_t need = plan(nullptr, *cfg, nullptr);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < need)
    return FLINT_ERR_WORKSPACE;
  flint_moe_ctx* h = new (std::nothrow) flint_moe_ctx();
  if (!h) return FLINT_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->w = w;
  h->ws = static_cast<char*>(workspace);
  h->ws_bytes = workspace_bytes;
  plan(h, *cfg, h->ws);
  h->last_T = 0;
  h->w4a4 = (cfg->flags & FLINT_FLAG_W4A4) != 0;
  const int n_wrows = cfg->n_slots > 0 ? cfg->n_slots : cfg->n_experts;   // experts (or slots) of the routed arrays
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaMemset(h->err, 0, 16) != cudaSuccess || cudaMemset(h->cnt, 0, kCntInts * 4) != cudaSuccess ||
      !encode_rows(&h->tm_gu, w.gu_codes, static_cast<uint64_t>(n_wrows) * 2 * kI, kH / 2, 64, 8) ||
      (cfg->fmt == FLINT_W_NVFP4 &&
       !encode_rows(&h->tm_gu_sc, w.gu_scales, static_cast<uint64_t>(n_wrows) * 2 * kI, kH / 16, 8, 8)) ||
      !encode_rows(&h->tm_sh_gu, w.sh_gu, 2 * kIs, kH * 2, 256, 2) ||
      !encode_rows(&h->tm_sh_dn, w.sh_dn, kH, kIs * 2, 64, 16) ||
      !encode_code_tiles(&h->tm_pf_gu, w.gu_codes, static_cast<uint64_t>(n_wrows) * 2 * kI, kH / 2) ||
      !encode_code_tiles(&h->tm_pf_dn, w.dn_codes, static_cast<uint64_t>(n_wrows) * kH, kI / 2) ||
      !encode_bf16_tiles(&h->tm_pf_sh_gu, w.sh_gu, 2 * kIs, kH) ||
      !encode_bf16_tiles(&h->tm_pf_sh_dn, w.sh_dn, kH, kIs) ||
      !encode_bf16_tiles(&h->tm_pf_router, w.router_w, cfg->n_experts, kH) ||
      !encode_bf16_tiles(&h->tm_pf_hs_hi, h->hs_hi, cfg->t_max, kIs) ||
      !encode_bf16_tiles(&h->tm_pf_hs_lo, h->hs_lo, cfg->t_max, kIs) ||
      !encode_f16_rows16(&h->tm_pf_xg, h->xg, static_cast<uint64_t>(cfg->t_max) * cfg->top_k, kH) ||
      !encode_f16_rows16(&h->tm_pf_hq, h->hq, static_cast<uint64_t>(cfg->t_max) * cfg->top_k, kI) ||
      !create_side_stream(h)) {
    delete h;
    return FLINT_ERR_CUDA;
  }
  if (h->w4a4) {
    const uint64_t P = static_cast<uint64_t>(cfg->t_max) * cfg->top_k;
    if (!encode_fp4_tiles(&h->tm_w4_gu, w.gu_codes, static_cast<uint64_t>(n_wrows) * 2 * kI, kH / 2, 128) ||
        !encode_fp4_tiles(&h->tm_w4_dn, w.dn_codes, static_cast<uint64_t>(n_wrows) * kH, kI / 2, 128) ||
        !encode_fp4_tiles(&h->tm_w4_xa, h->xa, P, kH / 2, 16) || !encode_fp4_tiles(&h->tm_w4_ha, h->ha, P, kI / 2, 16) ||
        // the weight scales in the MMA's layout, once (the weights' own writes complete first)
        cudaDeviceSynchronize() != cudaSuccess ||
        launch_pack_sf_atoms(static_cast<const uint8_t*>(w.gu_scales), n_wrows * 2 * kI, kH, h->w_atoms_gu, 0) !=
            cudaSuccess ||
        launch_pack_sf_atoms(static_cast<const uint8_t*>(w.dn_scales), n_wrows * kH, kI, h->w_atoms_dn, 0) !=
            cudaSuccess ||
        cudaStreamSynchronize(0) != cudaSuccess) {
      delete h;
      return FLINT_ERR_CUDA;
    }
  }
  // the decode kernel keeps every CTA resident (one per SM) and gives each at most 16 rows of y
  int per_sm = 0;
  if (decode_check_residency(cfg->fmt == FLINT_W_INT4_G128_FWHT128 ? kInt4 : kNvfp4, &per_sm) != cudaSuccess) {
    delete h;
    return FLINT_ERR_CUDA;
  }
  if (per_sm < 1 || h->n_sm < kH / 16) {
    delete h;
    return FLINT_ERR_UNSUPPORTED;
  }
  *out = h;
  return FLINT_OK;
}

flint_status flint_moe_forward(flint_moe_t h, const void* x, int T, void* y, void* stream) {
  if (!h || h->cfg.n_slots > 0) return FLINT_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.t_max) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!aligned16(x) || !aligned16(y) || x == y) return FLINT_ERR_INVALID_ARG;
  flint_status st = run_forward(h, static_cast<const uint16_t*>(x), T, static_cast<uint16_t*>(y),
                                static_cast<cudaStream_t>(stream));
  if (st == FLINT_OK) h->last_T = T;
  return st;
}

flint_status flint_moe_forward_host(flint_moe_t h, const void* x_host, int T, void* y_host, void* stream) {
  if (!h || h->cfg.n_slots > 0) return FLINT_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.t_max) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!x_host || !y_host) return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * kH * 2;
  FLINT_TRY(cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
  flint_status st = run_forward(h, h->x_stage, T, h->y_stage, s);
  if (st != FLINT_OK) return st;
  h->last_T = T;
  FLINT_TRY(cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, s));
  return FLINT_OK;
}

flint_status flint_moe_forward_routed(flint_moe_t h, const void* x, int T, const int* ids, const float* w, void* y,
                                      void* stream) {
  if (!h || h->cfg.n_slots > 0) return FLINT_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.t_max) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!aligned16(x) || !aligned16(y) || x == y || !ids || !w) return FLINT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ids) & 3u) || (reinterpret_cast<uintptr_t>(w) & 3u)) return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t P = static_cast<size_t>(T) * h->cfg.top_k;
  FLINT_TRY(cudaMemcpyAsync(h->ids, ids, P * 4, cudaMemcpyDeviceToDevice, s));
  FLINT_TRY(cudaMemcpyAsync(h->wts, w, P * 4, cudaMemcpyDeviceToDevice, s));
  flint_status st = run_forward(h, static_cast<const uint16_t*>(x), T, static_cast<uint16_t*>(y), s, true);
  if (st == FLINT_OK) h->last_T = T;
  return st;
}

flint_status flint_residual_rmsnorm(float* x, const void* y, int T, float eps, void* z, void* stream) {
  if (T < 0 || !(eps > 0.f)) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!aligned16(x) || (y && !aligned16(y)) || (z && !aligned16(z))) return FLINT_ERR_INVALID_ARG;
  FLINT_TRY(launch_residual_rmsnorm(x, static_cast<const uint16_t*>(y), T, eps, static_cast<uint16_t*>(z),
                                    static_cast<cudaStream_t>(stream)));
  return FLINT_OK;
}

flint_status flint_moe_stack_forward(const flint_moe_t* layers, int n_layers, float* x, int T, float eps, void* z,
                                     void* y, void* stream) {
  if (!layers || n_layers < 1 || T < 0 || !(eps > 0.f)) return FLINT_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!layers[l] || T > layers[l]->cfg.t_max || layers[l]->cfg.n_slots > 0) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!aligned16(x) || !aligned16(z) || !aligned16(y) || z == y) return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* zb = static_cast<uint16_t*>(z);
  uint16_t* yb = static_cast<uint16_t*>(y);
  for (int l = 0; l < n_layers; ++l) {
    FLINT_TRY(launch_residual_rmsnorm(x, l ? yb : nullptr, T, eps, zb, s));
    flint_status st = run_forward(layers[l], zb, T, yb, s);
    if (st != FLINT_OK) return st;
    layers[l]->last_T = T;
  }
  FLINT_TRY(launch_residual_rmsnorm(x, yb, T, eps, nullptr, s));
  return FLINT_OK;
}

flint_status flint_moe_routing(flint_moe_t h, int* ids, float* w, int* offsets, int* perm, void* stream) {
  if (!h) return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t P = static_cast<size_t>(h->last_T) * h->cfg.top_k;
  if (ids && P) FLINT_TRY(cudaMemcpyAsync(ids, h->ids, P * 4, cudaMemcpyDeviceToDevice, s));
  if (w && P) FLINT_TRY(cudaMemcpyAsync(w, h->wts, P * 4, cudaMemcpyDeviceToDevice, s));
  if (offsets) FLINT_TRY(cudaMemcpyAsync(offsets, h->offsets, (h->cfg.n_experts + 1) * 4, cudaMemcpyDeviceToDevice, s));
  if (perm && P) FLINT_TRY(cudaMemcpyAsync(perm, h->perm, P * 4, cudaMemcpyDeviceToDevice, s));
  return FLINT_OK;
}

flint_status flint_moe_intermediate(flint_moe_t h, int which, void* dst, size_t bytes, void* stream) {
  if (!h || !dst) return FLINT_ERR_INVALID_ARG;
  const size_t T = h->last_T;
  const void* src = nullptr;
  size_t have = 0;
  switch (which) {
    case FLINT_BUF_LOGITS: src = h->logits; have = T * h->cfg.n_experts * 4; break;
    case FLINT_BUF_XQ:
      if (T <= kDecodeMaxT) {
        src = h->xq;
        have = T * kH * 2;
      } else {
        src = h->xg;
        have = T * h->cfg.top_k * kH * 2;
      }
      break;
    case FLINT_BUF_YS: src = h->ys; have = T * kH * 4; break;
    case FLINT_BUF_XA: case FLINT_BUF_XA_SF: case FLINT_BUF_XA_TS: case FLINT_BUF_H:
    case FLINT_BUF_HA: case FLINT_BUF_HA_SF: case FLINT_BUF_HA_TS: case FLINT_BUF_O: {
      if (!h->w4a4 || T <= kDecodeMaxT) return FLINT_ERR_INVALID_ARG;
      const size_t P = T * h->cfg.top_k;
      const void* const srcs[] = {h->xa, h->xa_sf, h->xa_ts, h->h32, h->ha, h->ha_sf, h->ha_ts, h->o};
      const size_t sizes[] = {P * kH / 2, P * kH / 16, P * 4, P * kI * 4, P * kI / 2, P * kI / 16, P * 4, P * kH * 2};
      src = srcs[which - FLINT_BUF_XA];
      have = sizes[which - FLINT_BUF_XA];
      break;
    }
    default: return FLINT_ERR_INVALID_ARG;
  }
  if (bytes > have) return FLINT_ERR_INVALID_ARG;
  if (bytes) FLINT_TRY(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return FLINT_OK;
}

flint_status flint_moe_error_word(flint_moe_t h, unsigned* out) {
  if (!h || !out) return FLINT_ERR_INVALID_ARG;
  // the handle's own stream may still run part of a forward; the caller's stream must be idle
  if (h->side) FLINT_TRY(cudaStreamSynchronize(h->side));
  FLINT_TRY(cudaMemcpy(out, h->err, sizeof(unsigned), cudaMemcpyDeviceToHost));
  FLINT_TRY(cudaMemset(h->err, 0, sizeof(unsigned)));
  // a forward whose grid barrier gave up leaves its barrier words behind: start the next one clean
  if (*out & kErrTimeout) FLINT_TRY(cudaMemset(h->cnt, 0, kCntInts * 4));
  return FLINT_OK;
}

flint_status flint_moe_set_stage_events(flint_moe_t h, void* const* events, int n) {
  if (!h) return FLINT_ERR_INVALID_ARG;
  if (!events) {
    h->n_events = 0;
    return FLINT_OK;
  }
  if (n < 1 || n > 32) return FLINT_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!events[i]) return FLINT_ERR_INVALID_ARG;
    h->events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  h->n_events = n;
  return FLINT_OK;
}

int flint_moe_stage_count(flint_moe_t h, int T) { return h ? stage_count(h, T) : 0; }

const char* flint_moe_stage_name(flint_moe_t h, int T, int i) { return h ? stage_name(h, T, i) : nullptr; }

flint_status flint_moe_destroy(flint_moe_t h) {
  delete h;
  return FLINT_OK;
}

const char* flint_moe_status_string(flint_status s) {
  switch (s) {
    case FLINT_OK: return "ok";
    case FLINT_ERR_INVALID_ARG: return "invalid argument";
    case FLINT_ERR_UNSUPPORTED: return "unsupported shape or format";
    case FLINT_ERR_CUDA: return "CUDA error";
    case FLINT_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FLINT_ERR_DEVICE_CHECK: return "device-side check failed";
    case FLINT_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"

// ------------------------------------------------------------------------------- expert cache

struct flint_expert_cache {
  flint_moe_t layer;
  flint_moe_weights host;                  // routed weights of all E experts, host memory [E][...]
  size_t b_gu_codes, b_gu_scales, b_dn_codes, b_dn_scales;   // bytes per expert
  std::vector<int> slot_of, expert_of;
  std::vector<unsigned long long> last_use;
  unsigned long long tick;
  std::vector<int> ids, loads;
  long long hits, misses, bytes;
};

extern "C" int flint_cache_plan(int E, int S, int* slot_of, int* expert_of, unsigned long long* last_use,
                                unsigned long long tick, const int* ids, int P, int* loads) {
  if (E < 1 || S < 1 || !slot_of || !expert_of || !last_use || (P > 0 && !ids) || !loads) return -1;
  // distinct ids in order of first appearance, checked before anything changes
  std::vector<int> uniq;
  std::vector<char> seen(static_cast<size_t>(E), 0);
  for (int q = 0; q < P; ++q) {
    const int e = ids[q];
    if (e < 0 || e >= E) return -1;
    if (!seen[e]) {
      seen[e] = 1;
      uniq.push_back(e);
    }
  }
  if (static_cast<int>(uniq.size()) > S) return -1;
  for (int e : uniq)                       // hits keep their slots
    if (slot_of[e] >= 0) last_use[slot_of[e]] = tick;
  int n = 0;
  for (int e : uniq) {
    if (slot_of[e] >= 0) continue;
    int v = -1;
    for (int sl = 0; sl < S && v < 0; ++sl)
      if (expert_of[sl] < 0) v = sl;       // a free slot
    if (v < 0)                             // else the least recently used slot this forward does not need
      for (int sl = 0; sl < S; ++sl)
        if (last_use[sl] != tick && (v < 0 || last_use[sl] < last_use[v])) v = sl;
    if (expert_of[v] >= 0) slot_of[expert_of[v]] = -1;
    expert_of[v] = e;
    slot_of[e] = v;
    last_use[v] = tick;
    loads[2 * n] = e;
    loads[2 * n + 1] = v;
    ++n;
  }
  return n;
}

extern "C" {

flint_status flint_cache_create(flint_moe_t layer, const flint_moe_weights* host, flint_cache_t* out) {
  if (!out) return FLINT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!layer || !host || layer->cfg.n_slots <= 0) return FLINT_ERR_INVALID_ARG;
  const flint_moe_cfg& c = layer->cfg;
  if (!host->gu_codes || !host->gu_scales || !host->dn_codes || !host->dn_scales) return FLINT_ERR_INVALID_ARG;
  if (c.fmt == FLINT_W_NVFP4 && (!host->gu_tscale || !host->dn_tscale)) return FLINT_ERR_INVALID_ARG;
  if ((host->gu_tscale != nullptr) != (layer->w.gu_tscale != nullptr) ||
      (host->dn_tscale != nullptr) != (layer->w.dn_tscale != nullptr))
    return FLINT_ERR_INVALID_ARG;
  flint_expert_cache* k = new (std::nothrow) flint_expert_cache();
  if (!k) return FLINT_ERR_INVALID_ARG;
  const bool i4 = c.fmt == FLINT_W_INT4_G128_FWHT128;
  k->layer = layer;
  k->host = *host;
  k->b_gu_codes = static_cast<size_t>(2 * kI) * (kH / 2);
  k->b_gu_scales = i4 ? static_cast<size_t>(2 * kI) * (kH / kGroup) * 2 : static_cast<size_t>(2 * kI) * (kH / 16);
  k->b_dn_codes = static_cast<size_t>(kH) * (kI / 2);
  k->b_dn_scales = i4 ? static_cast<size_t>(kH) * (kI / kGroup) * 2 : static_cast<size_t>(kH) * (kI / 16);
  k->slot_of.assign(c.n_experts, -1);
  k->expert_of.assign(c.n_slots, -1);
  k->last_use.assign(c.n_slots, 0);
  k->tick = 0;
  k->ids.assign(static_cast<size_t>(c.t_max) * c.top_k, 0);
  k->loads.assign(2 * static_cast<size_t>(c.n_slots), 0);
  k->hits = k->misses = k->bytes = 0;
  *out = k;
  return FLINT_OK;
}

flint_status flint_cache_destroy(flint_cache_t c) {
  delete c;
  return FLINT_OK;
}

flint_status flint_cache_stats(flint_cache_t c, long long* hits, long long* misses, long long* bytes) {
  if (!c) return FLINT_ERR_INVALID_ARG;
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (bytes) *bytes = c->bytes;
  return FLINT_OK;
}

flint_status flint_moe_forward_cached(flint_moe_t h, flint_cache_t k, const void* x, int T, void* y, void* stream) {
  if (!h || !k || k->layer != h) return FLINT_ERR_INVALID_ARG;
  const flint_moe_cfg& c = h->cfg;
  if (T < 0 || T > c.t_max) return FLINT_ERR_INVALID_ARG;
  if (T == 0) return FLINT_OK;
  if (!aligned16(x) || !aligned16(y) || x == y) return FLINT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = c.n_experts, K = c.top_k, P = T * K;
  // routing on the device, ids back to the host
  FLINT_TRY(launch_router_logits(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(h->w.router_w), T, E,
                                 h->logits, s));
  FLINT_TRY(launch_topk(h->logits, 1, nullptr, T, E, K, c.norm_floor, h->ids, h->wts, c.flags, h->err, s));
  FLINT_TRY(cudaMemcpyAsync(k->ids.data(), h->ids, static_cast<size_t>(P) * 4, cudaMemcpyDeviceToHost, s));
  FLINT_TRY(cudaStreamSynchronize(s));
  // slots for the selected experts; copies of the misses
  const int n = flint_cache_plan(E, c.n_slots, k->slot_of.data(), k->expert_of.data(), k->last_use.data(), ++k->tick,
                                 k->ids.data(), P, k->loads.data());
  if (n < 0) return FLINT_ERR_UNSUPPORTED;
  int distinct = 0;
  for (int sl = 0; sl < c.n_slots; ++sl) distinct += k->last_use[sl] == k->tick;
  k->hits += distinct - n;
  k->misses += n;
  for (int i = 0; i < n; ++i) {
    const size_t e = static_cast<size_t>(k->loads[2 * i]), v = static_cast<size_t>(k->loads[2 * i + 1]);
    auto copy = [&](const void* dev_base, const void* host_base, size_t bytes) -> cudaError_t {
      k->bytes += static_cast<long long>(bytes);
      return cudaMemcpyAsync(static_cast<char*>(const_cast<void*>(dev_base)) + v * bytes,
                             static_cast<const char*>(host_base) + e * bytes, bytes, cudaMemcpyHostToDevice, s);
    };
    FLINT_TRY(copy(h->w.gu_codes, k->host.gu_codes, k->b_gu_codes));
    FLINT_TRY(copy(h->w.gu_scales, k->host.gu_scales, k->b_gu_scales));
    FLINT_TRY(copy(h->w.dn_codes, k->host.dn_codes, k->b_dn_codes));
    FLINT_TRY(copy(h->w.dn_scales, k->host.dn_scales, k->b_dn_scales));
    if (h->w.gu_tscale) FLINT_TRY(copy(h->w.gu_tscale, k->host.gu_tscale, 2 * sizeof(float)));
    if (h->w.dn_tscale) FLINT_TRY(copy(h->w.dn_tscale, k->host.dn_tscale, sizeof(float)));
  }
  // the slot map (pageable source: the driver stages it before the call returns)
  FLINT_TRY(cudaMemcpyAsync(h->slot_of, k->slot_of.data(), static_cast<size_t>(E) * 4, cudaMemcpyHostToDevice, s));
  flint_status st = run_forward(h, static_cast<const uint16_t*>(x), T, static_cast<uint16_t*>(y), s, true);
  if (st == FLINT_OK) h->last_T = T;
  return st;
}

}  // extern "C"
