/*
 * plx_synth.h — C ABI of libplx_synth.so: the seeded synthetic-input generator
 * on the device.  It holds no Parallax arithmetic; it exists so that multi-GB
 * KV caches can be filled in place with exactly the values that the host-side
 * generator (local_linear_attention_streamed_b200/synth.py) produces for any
 * slice the float64 oracle checks.
 *
 * Generator: element c of a tensor takes h = SplitMix64 output number c of the
 * stream seeded by `key` (Steele, Lea and Flood, OOPSLA 2014), n = sum of the
 * four 16-bit lanes of h - 2*65535, then
 *   dist 0 (NORMAL):   value = (double)n * scale
 *   dist 1 (RMS_ROWS): value = (double)n / sqrt(sum_row(n^2) / row)   (exact int64 row sum)
 * rounded double -> float (nearest even), and for bf16 float -> bf16 (nearest even).
 */
#ifndef PLX_SYNTH_H
#define PLX_SYNTH_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Fills `count` elements at device pointer `dst` (dtype 0 = f32, 1 = bf16),
 * asynchronously on `stream` (void* stands for cudaStream_t).  For dist 1,
 * `row` is the row length and must divide `count`.  Returns 0, -1 for a bad
 * argument, -4 for a CUDA launch failure.
 */
int plx_synth_fill(void* dst, int dtype, uint64_t key, uint64_t count, int dist, double scale,
                   int64_t row, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PLX_SYNTH_H */
