/*
 * synth.h -- seeded, counter-based synthetic input generator.
 *
 * This module produces the input tensors (hidden states, gate weight,
 * correction bias, expert weights) for every workload of the MoE layer.  It
 * contains none of the layer's arithmetic: it only maps
 * (seed, tensor id, element index) to a value, identically on the host and on
 * the GPU, so that the CPU reference and the CUDA library can be fed the same
 * bits without either of them importing the other.
 *
 * Definition (both twins implement exactly this):
 *   gamma      = 0x9E3779B97F4A7C15
 *   mix64(z)   = the SplitMix64 output function:
 *                z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   key        = mix64(mix64(seed + gamma) + (tensor_id + 1) * gamma)
 *   draw(i, j) = mix64(key + (2*i + j + 1) * gamma)          (i: element, j: 0/1)
 *
 *   normal(i)  : the eight 16-bit fields of draw(i,0) and draw(i,1) are summed
 *                as integers (Irwin-Hall with n = 8), centred by subtracting
 *                8 * 65535 / 2 = 262140, converted to fp32 (exact, the
 *                magnitude is below 2^24), multiplied in fp32 by
 *                SYNTH_IH8_SCALE (1 / std of the integer sum), then by sigma.
 *                Two correctly rounded fp32 multiplies, no FMA, no libm.
 *                bf16 tensors round that fp32 value to nearest-even.
 *   uniform(i) : t = (float)(draw(i,0) >> 40) * 2^-24   (exact)
 *                value = lo + (hi - lo) * t, three correctly rounded fp32 ops.
 *
 * Every value depends only on its own index, so any slice of a tensor (one
 * expert's weights, one token's row) can be regenerated on its own.
 */
#ifndef SYNTH_H
#define SYNTH_H

#include <stdint.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL
#define SYNTH_M1 0xBF58476D1CE4E5B9ULL
#define SYNTH_M2 0x94D049BB133111EBULL
/* 1 / sqrt(8 * (65536^2 - 1) / 12), rounded to fp32. */
#define SYNTH_IH8_SCALE 0x1.3988e2p-16f /* 1.8688124e-05 */
#define SYNTH_IH8_CENTER 262140

#endif
