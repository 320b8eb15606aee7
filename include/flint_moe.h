/*
 * flint_moe.h - C ABI of a B200 (sm_100a) forward pass of one Flint mixture-of-experts layer.
 *
 * The layer (Aijuus/flint-w4exp, model summary; midagedev/bloomery issue #632, description;
 * WaveCut/Flint-UD-Q4_K_XL-NInfer-v3 README, "What is inside"):
 *
 *   logits[t,e] = sum_j W_r[e,j] x[t,j]                       fp32 accumulation of exact bf16 products
 *   s = sigmoid(logits); pick the top_k experts by score (no correction bias; ties to the lower id);
 *   list the slots by ascending expert id; w_k = s_k / max(sum_k s_k, norm_floor)
 *   routed expert e:  h = silu(Wg_e x') * (Wu_e x');  o = Wd_e h'
 *   shared expert:    hs = silu(Sg x) * (Su x);       ys = Sd hs
 *   y[t] = bf16( routed_scale * sum_k w_k o_k + ys )  (fixed slot order, one final rounding)
 *
 * For the int4 format x' and h' are x and h rotated per 128-segment by the normalised Sylvester
 * Hadamard matrix Hn = H_128/sqrt(128) (the codes store W * blockdiag(Hn), Aijuus/flint-w4exp,
 * weights row). For NVFP4, x' = x and h' = h (kekzle/Flint-NVFP4, W4A16).
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument that names layer data is a DEVICE pointer owned by the caller; the
 *    library only borrows it and never allocates, frees or copies it. It must stay valid while
 *    the handle uses it. Host pointers are named *_host.
 *  - Device pointers must be 16-byte aligned; a misaligned or NULL pointer is rejected with
 *    FLINT_ERR_INVALID_ARG before anything is launched.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Work is enqueued
 *    asynchronously; no call synchronises the stream unless it says so.
 *  - A handle is not re-entrant: its workspace holds one forward at a time, so calls on one
 *    handle from several streams must be ordered by the caller.
 *  - bf16 tensors are passed as raw 16-bit patterns (uint16_t or __nv_bfloat16 storage).
 */
#ifndef FLINT_MOE_H
#define FLINT_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum flint_status {
  FLINT_OK = 0,
  FLINT_ERR_INVALID_ARG = 1,   /* NULL/misaligned pointer, T out of range, bad cfg value */
  FLINT_ERR_UNSUPPORTED = 2,   /* a shape or format this build has no kernels for */
  FLINT_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
  FLINT_ERR_WORKSPACE = 4,     /* workspace NULL, misaligned or smaller than flint_moe_workspace_size */
  FLINT_ERR_DEVICE_CHECK = 5,  /* a device-side check set the handle's error word */
  FLINT_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up */
} flint_status;

typedef enum flint_wformat {
  /* int4 two's-complement codes, two per byte along K (low nibble = even K), one bf16 scale per
   * 128 of K, stored against the per-128 Hadamard rotation (Aijuus/flint-w4exp, weights row). */
  FLINT_W_INT4_G128_FWHT128 = 0,
  /* NVFP4: E2M1 codes two per byte (low nibble = even column), one E4M3 (fn) scale per 16
   * columns, one F32 tensor scale per Linear (kekzle/Flint-NVFP4, "What is in the files"). */
  FLINT_W_NVFP4 = 1
} flint_wformat;

/* cfg.flags */
#define FLINT_FLAG_DEBUG_CHECKS 0x1u  /* device-side range checks on ids / offsets; sets the error word */
/* W4A4 prefill (FLINT_W_NVFP4 only; forwards with T > 8): the routed experts' inputs, x and the
 * SwiGLU output h, are quantised to NVFP4 per row before each projection, and the projections run
 * as block-scaled FP4 MMAs (kekzle/Flint-NVFP4, evaluation table and serving notes: imp quantises
 * activations in prefill). Per row: a tensor scale amax / (6 * 448) (1 for an all-zero row), an E4M3
 * scale per 16 values (nearest, ties to even, saturating), E2M1 codes (nearest, ties to even), each
 * quotient and product rounded to fp32 in that order. Decode (T <= 8) keeps 16-bit activations.
 * flint_moe_create copies the weight block scales into the MMA's layout (workspace; it synchronises
 * the device first), so the weights must not change while the handle lives; not with n_slots > 0
 * (FLINT_ERR_UNSUPPORTED). Adds ~60 MB to the workspace at E = 256, t_max = 2048 (scale atoms of
 * the weights, and NVFP4 rows of x and h with their atoms, ~1.8 KB per permuted row). */
#define FLINT_FLAG_W4A4 0x2u

typedef struct flint_moe_cfg {
  int hidden;         /* H: 2048 (the only width this build has kernels for) */
  int n_experts;      /* E: a multiple of 32 in [32, 256] (Flint: 256) */
  int top_k;          /* experts per token, 1..8 (Flint: 6) */
  int inter;          /* I, routed SwiGLU width: 512 */
  int inter_shared;   /* Is, shared-expert SwiGLU width: 1024 */
  int fmt;            /* flint_wformat */
  int t_max;          /* largest token count forward() will be given, 1..16384 */
  float routed_scale; /* multiplies the routed sum (Flint: 1.0) */
  float norm_floor;   /* floor of the selected-score sum (Flint: 2^-14) */
  unsigned flags;     /* FLINT_FLAG_* */
  int n_slots;        /* 0: the routed experts' weights are device arrays over all E experts. > 0: they
                         are n_slots device slots of an expert cache (n_slots <= E), filled from host
                         memory by flint_moe_forward_cached, the only forward such a handle takes */
} flint_moe_cfg;

/* Weight pointers (device, caller-owned, row-major [out][in]).
 *   router_w   bf16 [E][H]
 *   gu_codes   u8   [E][2I][H/2]   rows 0..I-1 are the gate projection, rows I..2I-1 the up projection
 *   gu_scales  int4: bf16 [E][2I][H/128]; nvfp4: E4M3 [E][2I][H/16]
 *   gu_tscale  f32  [E][2] (gate, up) tensor scales; required for nvfp4, optional (NULL = 1) for int4
 *   dn_codes   u8   [E][H][I/2]
 *   dn_scales  int4: bf16 [E][H][I/128]; nvfp4: E4M3 [E][H][I/16]
 *   dn_tscale  f32  [E]; required for nvfp4, optional (NULL = 1) for int4
 *   sh_gu      bf16 [2*Is][H]   gate rows then up rows
 *   sh_dn      bf16 [H][Is]
 * The int4 path multiplies codes by their bf16 scale in fp16, which is exact while
 * 2^-14 <= |scale| <= 8188; out-of-range scales can be brought in range with a power of two folded
 * into gu_tscale / dn_tscale (applied in fp32). */
typedef struct flint_moe_weights {
  const void* router_w;
  const void* gu_codes;
  const void* gu_scales;
  const float* gu_tscale;
  const void* dn_codes;
  const void* dn_scales;
  const float* dn_tscale;
  const void* sh_gu;
  const void* sh_dn;
} flint_moe_weights;

typedef struct flint_moe_ctx* flint_moe_t;

/* Bytes of device workspace a handle with this cfg needs (0 if cfg is invalid). Depends on
 * t_max, E, top_k and the widths only. */
size_t flint_moe_workspace_size(const flint_moe_cfg* cfg);

/* Validates cfg and the weight pointers, and records them with the caller's workspace (device,
 * 256-byte aligned, at least flint_moe_workspace_size bytes, owned by the caller). Allocates no
 * device memory; its only device work is two synchronous cudaMemsets that clear the handle's
 * 16-byte error word and its arrival counters inside the workspace. It creates one non-blocking
 * stream and two events of its own (released by flint_moe_destroy), on which forward() runs part
 * of a T > 8 forward. On success *out receives a handle. */
flint_status flint_moe_create(const flint_moe_cfg* cfg, const flint_moe_weights* weights, void* workspace,
                              size_t workspace_bytes, flint_moe_t* out);

/* y = MoE(x) for T tokens: x bf16 [T][H] and y bf16 [T][H] are device pointers (distinct buffers).
 * 0 <= T <= t_max (T = 0 is a no-op). Enqueues the kernels on `stream` and returns; the host never
 * waits and nothing is copied back. T <= 8 takes the decode path: three kernels (route, gate|up,
 * down + combine) chained by programmatic dependent launch, so each one starts streaming weights
 * before its predecessor ends. Larger T takes the tensor-core path: the routing chain (router,
 * top-k, permutation, activation operand) runs on the handle's own stream, forked from and joined
 * back into `stream` with events (so graph capture of `stream` captures it too), while the shared
 * expert runs on `stream`; then the routed gate|up and down grouped GEMMs and the combine. */
flint_status flint_moe_forward(flint_moe_t h, const void* x, int T, void* y, void* stream);

/* As flint_moe_forward, with x_host and y_host in host memory (pinned memory gives asynchronous
 * copies): copies x into the workspace, runs the forward and copies y back, all on `stream`.
 * The caller synchronises the stream before reading y_host. */
flint_status flint_moe_forward_host(flint_moe_t h, const void* x_host, int T, void* y_host, void* stream);

/* As flint_moe_forward, with the routing given instead of computed: ids int32 [T][top_k] (device,
 * distinct expert ids in [0, E), ascending within a token) and w f32 [T][top_k] (device), e.g. from
 * flint_moe_route_noalloc or another router. The layer then runs its permutation, experts and
 * combine on that routing (ids out of range are clamped). */
flint_status flint_moe_forward_routed(flint_moe_t h, const void* x, int T, const int* ids, const float* w, void* y,
                                      void* stream);

/* Host-resident routed experts with a device cache of hot experts (WaveCut/Flint-UD-Q4_K_XL-NInfer-v3
 * README, "Running": the routed experts may live in host memory; "Memory": per-layer expert banks).
 * The layer handle is created with cfg.n_slots = S > 0 and its routed weight pointers at S device
 * slots ([S][...] in the same per-expert layout as the [E][...] arrays); `host` holds the routed
 * weights of all E experts in HOST memory ([E][...], page-locked so that the copies run
 * asynchronously; router_w, sh_gu and sh_dn are not used). The cache keeps which expert sits in which
 * slot and replaces the least recently used expert that the current forward does not need. Host
 * memory only: the cache object allocates no device memory. */
typedef struct flint_expert_cache* flint_cache_t;
flint_status flint_cache_create(flint_moe_t layer, const flint_moe_weights* host, flint_cache_t* out);
flint_status flint_cache_destroy(flint_cache_t c);
/* hits and misses count expert loads (one per distinct expert of a forward); bytes = host-to-device
 * bytes copied into slots. Any pointer may be NULL. */
flint_status flint_cache_stats(flint_cache_t c, long long* hits, long long* misses, long long* bytes);

/* y = MoE(x) with the routed experts in host memory: the routing runs on the device (router logits and
 * top-k), the selected ids are read back (this call SYNCHRONISES `stream` once, mid-forward), every
 * selected expert not in a slot is copied into one (cudaMemcpyAsync on `stream`), the slot map is
 * uploaded and the forward runs on that routing with the weights read from the slots. More distinct
 * selected experts than slots: FLINT_ERR_UNSUPPORTED, nothing enqueued beyond the routing. */
flint_status flint_moe_forward_cached(flint_moe_t h, flint_cache_t c, const void* x, int T, void* y, void* stream);

/* The cache's replacement rule as a pure host function (no CUDA call; exposed for tests and for
 * callers that manage slots themselves). State: slot_of [E] (slot of each expert or -1), expert_of [S]
 * (expert in each slot or -1), last_use [S] (tick of each slot's last use). ids [P] are the selected
 * experts of one forward at time `tick` (> every last_use). Every distinct id gets a slot: a hit keeps
 * its slot; a miss takes a free slot, else the slot with the smallest last_use among slots not used at
 * `tick`; the state is updated. loads [2*S] receives (expert, slot) pairs of the misses in the order
 * their ids first appear. Returns the number of misses, or -1 (state unchanged) when the distinct ids
 * exceed S or an id is out of range. */
int flint_cache_plan(int E, int S, int* slot_of, int* expert_of, unsigned long long* last_use, unsigned long long tick,
                     const int* ids, int P, int* loads);

/* Residual stream step of a stack of layers (the model's routed blocks with their weightless
 * RMSNorm; Aijuus/flint-w4exp, model summary): x f32 [T][H] (device, in/out) += y bf16 [T][H] when y is
 * not NULL; then, when z is not NULL, z bf16 [T][H] = bf16( x / sqrt(mean_j x[t][j]^2 + eps) ) per token,
 * the sum of squares reduced in a fixed order. One kernel, enqueued on `stream`. */
flint_status flint_residual_rmsnorm(float* x, const void* y, int T, float eps, void* z, void* stream);

/* n_layers layers in sequence on the residual x f32 [T][H] (device, in/out):
 *   for each layer l: z = bf16(rmsnorm(x)); y = layer_l(z); x += y
 * (the residual add of one layer is fused with the RMSNorm of the next). z and y are caller-owned
 * bf16 [T][H] scratch buffers (distinct). The handles must not run forwards concurrently. Each
 * layer's forward is the same launch sequence as flint_moe_forward; T <= every layer's t_max. */
flint_status flint_moe_stack_forward(const flint_moe_t* layers, int n_layers, float* x, int T, float eps, void* z,
                                     void* y, void* stream);

/* Device-to-device copies of the last forward's routing, enqueued on `stream` (any pointer may be
 * NULL to skip it): ids int32 [T][top_k] and w f32 [T][top_k] in slot order (ascending expert id),
 * offsets int32 [E+1] (exclusive prefix of per-expert counts), perm int32 [T*top_k] (position p
 * holds t*top_k+k, ordered by expert then token). */
flint_status flint_moe_routing(flint_moe_t h, int* ids, float* w, int* offsets, int* perm, void* stream);

/* Intermediates of the last forward, for tests: device-to-device copy of `bytes` bytes. */
enum {
  FLINT_BUF_LOGITS = 0,   /* f32 [T][E] router logits */
  FLINT_BUF_XQ = 1,       /* fp16, the routed experts' input: rotated x (int4) or x (nvfp4), each
                             8-element block stored in the order 0,4,1,5,2,6,3,7 for int4; [T][H]
                             after a forward with T <= 8, [T*top_k][H] in permuted row order (row p
                             holds token perm[p] / top_k) after a larger one */
  FLINT_BUF_YS = 2,       /* f32 [T][H] shared-expert output */
  /* W4A4 prefill only (FLINT_FLAG_W4A4, T > 8), permuted row order, P = T * top_k rows: */
  FLINT_BUF_XA = 3,       /* u8 [P][H/2] NVFP4 codes of x (low nibble = even column) */
  FLINT_BUF_XA_SF = 4,    /* u8 [P][H/16] their E4M3 block scales */
  FLINT_BUF_XA_TS = 5,    /* f32 [P] their tensor scales */
  FLINT_BUF_H = 6,        /* f32 [P][I] SwiGLU output h */
  FLINT_BUF_HA = 7,       /* u8 [P][I/2] NVFP4 codes of h */
  FLINT_BUF_HA_SF = 8,    /* u8 [P][I/16] */
  FLINT_BUF_HA_TS = 9,    /* f32 [P] */
  FLINT_BUF_O = 10        /* fp16 [P][H] routed expert outputs before weighting */
};
flint_status flint_moe_intermediate(flint_moe_t h, int which, void* dst, size_t bytes, void* stream);

/* Synchronously reads and clears the handle's device error word (set by device-side checks and
 * bounded waits). *out = 0 when nothing was flagged. */
flint_status flint_moe_error_word(flint_moe_t h, unsigned* out);

/* Instrumentation. With events != NULL every later forward records events[0] (a cudaEvent_t) on its
 * stream before its first kernel and events[i+1] after its i-th kernel, so consecutive events time
 * one kernel each; n must be at least flint_moe_stage_count(h, T) + 1 for the T used. The events are
 * caller-owned. events == NULL turns recording off. On the decode path an event between two
 * kernels removes their overlap, so per-kernel times then add up to more than an uninstrumented
 * forward. */
flint_status flint_moe_set_stage_events(flint_moe_t h, void* const* events, int n);

/* Number of kernels forward(h, ., T, .) launches, and the name of the i-th (NULL if out of range). */
int flint_moe_stage_count(flint_moe_t h, int T);
const char* flint_moe_stage_name(flint_moe_t h, int T, int i);

/* Routing without any caller-provided device memory beyond inputs and outputs (this entry point
 * has no counterpart in the published descriptions of the layer; it exists for callers that cannot
 * allocate: plug-ins whose host owns the allocator, loops that cannot afford the synchronisation an
 * allocation may cause).
 * Computes, for T tokens, the routing of flint_moe_forward: ids [T][top_k] (int32, ascending expert
 * id) and weights w [T][top_k] (f32). x bf16 [T][2048] and router_w bf16 [n_experts][2048] are
 * device inputs, ids and w device outputs, all caller-owned. Its fp32 logits come from the same
 * exact bf16 products as the forward's but are summed in another order, so the two agree to fp32
 * rounding of the logits: ids are equal unless two scores lie within a few fp32 ulps, and w to a few
 * ulps. The logits between its two kernels live in a fixed device array inside the library (64 KiB,
 * held on every GPU that loads the library until the process exits), so T <= 64 and n_experts <= 256
 * (a multiple of 32); larger sizes return FLINT_ERR_INVALID_ARG without launching anything. Calls no
 * cudaMalloc or cudaFree. The first call in a CUDA context looks up the array's device address (once
 * per device and context, with that device current); a context destroyed and re-created
 * (cudaDeviceReset) is noticed and the address looked up again. All calls share the one array:
 * calls whose kernels may overlap on the GPU (different streams without ordering) race on it and
 * must be serialised by the caller. */
flint_status flint_moe_route_noalloc(const void* x, const void* router_w, int T, int n_experts, int top_k,
                                     float norm_floor, int* ids, float* w, void* stream);

/* Frees the host-side handle only; the caller still owns weights and workspace. NULL is a no-op. */
flint_status flint_moe_destroy(flint_moe_t h);

/* Static description of a status code. */
const char* flint_moe_status_string(flint_status s);

#ifdef __cplusplus
}
#endif

#endif /* FLINT_MOE_H */
