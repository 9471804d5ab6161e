/*
 * dcu_gen.h -- device side of the seeded synthetic-input generator
 * (libdcugen.so).  Not part of the DCU method: it only produces the seeded
 * weights and token ids that the tests and the bench feed to libdcu, bit for
 * bit equal to the host implementation in dynamic_layer_wise_b200/inputs.py.
 *
 * Definition (arithmetic modulo 2^64):  base = mix((seed << 32) ^ tid);
 * h(i) = mix(base + (i + 1) * 0x9E3779B97F4A7C15), where mix is the
 * SplitMix64 finaliser (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014);  S = sum of the four 16-bit lanes of h;
 * value = (S - 131070) * ((std * sqrt(3)) / 65536) in binary64, then rounded
 * to bfloat16 (nearest-even on the binary64 bit pattern) or to float32.
 */
#ifndef DCU_GEN_H
#define DCU_GEN_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

/* out: dev [n] elements of dtype (0 = bf16, 1 = float32); element k gets the
 * value of index start + k of stream (seed, tid).  Returns 0 or -3 (CUDA error). */
int dcugen_normal(void *out, int64_t n, uint64_t seed, uint32_t tid, uint64_t start, double std, int32_t dtype,
                  void *stream);
/* out: dev [n] elements of dtype set to value.  Returns 0 or -3. */
int dcugen_fill(void *out, int64_t n, float value, int32_t dtype, void *stream);

#ifdef __cplusplus
}
#endif
#endif
