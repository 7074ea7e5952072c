/*
 * f16_selfcheck.c -- TEST INFRASTRUCTURE.  Pins the oracle's hand-written
 * binary32 -> binary16 conversion against an independent one: the host
 * compiler's _Float16 cast (IEEE 754 round to nearest, ties to even).
 * Counts the fp32 bit patterns p = start, start+stride, ... < stop on which
 * the two disagree (two NaNs count as agreeing; NaN payloads are not
 * compared).  Runs on all host threads (OpenMP).
 */
#include <stdint.h>
#include <string.h>

uint16_t or_f32_to_f16(float f);

int64_t or_f16_selfcheck(uint64_t start, uint64_t stop, uint64_t stride)
{
    int64_t bad = 0;
    if (stride == 0) stride = 1;
    int64_t count = (int64_t)((stop - start + stride - 1) / stride);
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = 0; i < count; i++) {
        uint32_t u = (uint32_t)(start + (uint64_t)i * stride);
        float f;
        memcpy(&f, &u, 4);
        _Float16 h = (_Float16)f;
        uint16_t ref;
        memcpy(&ref, &h, 2);
        uint16_t got = or_f32_to_f16(f);
        int ref_nan = (ref & 0x7C00u) == 0x7C00u && (ref & 0x3FFu);
        int got_nan = (got & 0x7C00u) == 0x7C00u && (got & 0x3FFu);
        if (ref_nan || got_nan) {
            if (ref_nan != got_nan) bad++;
        } else if (ref != got) {
            bad++;
        }
    }
    return bad;
}
