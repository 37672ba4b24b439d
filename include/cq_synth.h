/*
 * cq_synth.h -- device-side synthetic inputs for the large workloads (libcq_synth.so).
 *
 * Not part of the quantizer: these calls only fill buffers with seeded test data. They
 * implement the counter-based generator SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; the output function of Vigna's public
 * splitmix64.c): value i of stream (seed, stream_id) is the (i+1)-th SplitMix64 output from
 * the state key = mix(seed * 0x9E3779B97F4A7C15 + stream_id). Derived values use integer
 * operations and single binary32 multiplies only, so a host implementation of the same
 * definition reproduces them bit for bit. All pointers are device pointers owned by the
 * caller; calls are asynchronous on `stream`; the return value is 0 on success, 1 for a bad
 * argument, 7 for a CUDA launch error.
 */
#ifndef CQ_SYNTH_H
#define CQ_SYNTH_H

#include <stdint.h>

#include "cq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* stream identifiers */
#define CQS_STREAM_WEIGHT 1u
#define CQS_STREAM_CODE 2u
#define CQS_STREAM_SCALE 3u
#define CQS_STREAM_ZERO 4u
#define CQS_STREAM_RESID 5u

/* out[i] = float(d(first+i)) * mult, d = centred sum of the four 16-bit fields of the hash
 * (an Irwin-Hall(4) draw); mult = sigma / sqrt((65536^2 - 1) / 3) gives standard deviation sigma. */
int cqs_normal_f32(float *out, int64_t n, uint64_t seed, uint32_t stream_id, int64_t first,
                   float mult, cq_stream_t stream);

/* out[j] = hash(seed, CODE, first_word + j): 64-bit words of packed 4-bit codes. */
int cqs_code_words(uint64_t *out, int64_t n_words, uint64_t seed, int64_t first_word, cq_stream_t stream);

/* fp16 scale bits 0x1C00 | (hash(seed, SCALE, first+g) & 0x3FF): values in [2^-8, 2^-7). */
int cqs_scales(uint16_t *out, int64_t n, uint64_t seed, int64_t first, cq_stream_t stream);

/* zero points (hash(seed, ZERO, first+g) >> 20) & 15. */
int cqs_zeros(uint8_t *out, int64_t n, uint64_t seed, int64_t first, cq_stream_t stream);

/* bf16 residual bits RN_bf16(float(d(first+i)) * RN32(s_f * mult)) with s_f the fp16 scale of
 * element i's group: scale[i / 64] (scale covers this range; first % 64 == 0, n % 64 == 0). */
int cqs_residual_bf16(uint16_t *out, const uint16_t *scale, int64_t n, uint64_t seed, int64_t first,
                      float mult, cq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
