// kda_slots.h -- the per-(chunk, head) workspace slot that the chunk-local
// forward kernel writes and the chunk walks (forward and backward) read.
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace kda {

constexpr int CH = 64;    // chunk length
constexpr int DK = 128;   // key head dim
constexpr int DV = 128;   // value head dim
constexpr int DVS = 32;   // value columns per chain CTA
constexpr int NSL = DV / DVS;

// Workspace slot per (chunk, head), all offsets 16-byte aligned:
//   Mlr  bf16 K-major SW128 image [128 key rows][128 K]          32768 B
//   Qp   bf16 MN-major no-swizzle image, M = 64 tokens, K = 128   16384 B
//   GamC fp32 [128]                                                512 B
//   Bm   bf16 [4 slices][128 key rows][32 value cols]            32768 B
//   Ob   bf16 [4 slices][64 tokens][32 value cols]               16384 B
// In Bm and Ob the four 16-byte pieces of each 64-byte row r are stored in the
// order piece ^ ((r >> 1) & 3) (swz64), so that eight consecutive rows read or
// written 16 bytes at a time touch eight different bank groups.
// Element (row m, column i) of Mlr sits at (i >> 6) * 16384 + sw128_off(m, i & 63);
// element (token t, key channel i) of Qp at (t >> 3) * 128 + (i >> 3) * 1024 +
// (i & 7) * 16 + (t & 7) * 2.  Qp carries the output scale.
constexpr size_t SO_M = 0, SO_Q = 32768, SO_G = 49152, SO_B = 49664, SO_O = 82432;
constexpr size_t SLOT_BYTES = 98816;
constexpr uint32_t SO_MQG = 49664;         // Mlr + Qp + GamC, one contiguous copy
constexpr uint32_t BSL = DK * DVS * 2;     // one Bm slice, 8192 B
constexpr uint32_t OSL = CH * DVS * 2;     // one Ob slice, 4096 B

// A 128 x 128 state as a bf16 tensor-core operand image (the backward pass keeps its
// chunk-boundary states and chunk-end state gradients this way): element (row i,
// column j) at state_img_off(i, j), rows in 16-byte pieces of 8 columns, 8-row core
// matrices of 128 bytes, column pieces 128 bytes apart, row groups 2,048 bytes apart.
constexpr uint32_t STATE_IMG_BYTES = DK * DV * 2;
__host__ __device__ inline uint32_t state_img_off(uint32_t i, uint32_t j) {
    return (i >> 3) * 2048u + (j >> 3) * 128u + (i & 7u) * 16u + (j & 7u) * 2u;
}

}  // namespace kda
