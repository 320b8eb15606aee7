/* Weight preparation for the Flint MoE layer: the quantisers that turn bf16 expert weights into the
 * two routed-expert storage formats flint_moe_create takes (flint_moe.h, flint_wformat).
 *
 * int4 g128 with rotation (Aijuus/flint-w4exp, summary table, weights row: codes i4, group 128, bf16
 * scale, 128-wide Hadamard rotation; the container is converted from the bf16 checkpoint, same page,
 * "Serving it"). The stored matrix is W blockdiag(Hn), Hn = H_128 / sqrt(128), so every 128-segment
 * of a row is rotated and then rounded: per segment s = bf16(max|r| / 7) and code = clamp(rint(r * (1/s)),
 * -8, 7), 1/s the correctly rounded fp32 reciprocal.
 *
 * NVFP4 (kekzle/Flint-NVFP4, "What is in the files": E2M1 codes two per byte, E4M3 scale per 16
 * columns, F32 tensor scale per Linear; value = code x block scale x tensor scale): tensor scale =
 * amax / (6 * 448) (1 for an all-zero Linear); block scale = E4M3(block amax / (6 * tensor scale)),
 * nearest even, saturated at 448; code = E2M1(w * (1 / (block scale * tensor scale))), the reciprocal
 * correctly rounded in fp32; nearest grid value, ties to the even code, saturated at 6, sign from the
 * sign bit of the product.
 *
 * Every step is IEEE fp32 with one rounding per operation, in a fixed order (the rotation is the
 * Sylvester butterfly by stages 1, 2, 4, ..., 64 followed by one multiplication by the fp32 nearest
 * to 2^-3.5), so the codes do not depend on scheduling and can be checked bit for bit.
 *
 * Both functions enqueue kernels on `stream` and return; all pointers are device pointers owned by
 * the caller; nothing is allocated. Bad arguments return FLINT_ERR_INVALID_ARG before any launch. */
#ifndef FLINT_QUANT_H
#define FLINT_QUANT_H

#include "flint_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* w bf16 [rows][cols] (row-major, 16-byte aligned) -> codes u8 [rows][cols/2] (two's complement,
 * low nibble = even column; 2-byte aligned) and scales bf16 [rows][cols/128]. cols is a positive
 * multiple of 128, rows >= 0. rotate = 1 stores the rotated matrix (the layer's format), 0 the plain
 * one. A group whose values are all zero gets scale 0 and codes 0. */
flint_status flint_quantize_int4_g128(const void* w, long long rows, int cols, int rotate, void* codes, void* scales,
                                      void* stream);

/* n_mats Linears of rows x cols each, w bf16 [n_mats][rows][cols] (16-byte aligned) -> codes u8
 * [n_mats][rows][cols/2] (low nibble = even column; 8-byte aligned), scales E4M3 [n_mats][rows][cols/16]
 * and tscale f32 [n_mats] (4-byte aligned; used as scratch for the Linears' amax until the last of the
 * three kernels writes the tensor scales). cols is a positive multiple of 16; rows >= 1 unless n_mats
 * is 0. A routed gate|up bank [E][2I][H] is n_mats = 2E Linears of I rows (gate, then up, per expert),
 * so tscale comes out in the layer's [E][2] order. */
flint_status flint_quantize_nvfp4(const void* w, int n_mats, int rows, int cols, void* codes, void* scales,
                                  float* tscale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLINT_QUANT_H */
