// Counter-based N(0,1) stream on the device: splitmix64 + Box-Muller with this
// library's own ln / sin / cos.
//
// The pages keep LoZO's "random-direction stream" unchanged ("Zeroth-Order
// Fine-Tuning Was an Inference Workload All Along", section "The System
// Reorganization") without saying how it is drawn; this library fixes one
// counter-based definition so that every direction can be re-drawn from
// (seed, step, layer, matrix) anywhere, with no stored state:
//
//  * splitmix64 (Steele, Lea & Flood 2014; Vigna's public-domain finaliser):
//    the j-th output for key k is mix(k + (j+1) * 0x9E3779B97F4A7C15);
//  * Box-Muller on word b: u1 = ((b >> 40) + 1) 2^-24, u2 = (b & 0xFFFFFF) 2^-24,
//    z0 = sqrt(-2 ln u1) cos(2 pi u2), z1 = sqrt(-2 ln u1) sin(2 pi u2);
//  * ln m = 2 atanh((m-1)/(m+1)) summed to the s^11/11 term on
//    m in [sqrt(1/2), sqrt(2)), plus e ln 2 split in a high part (low 8 bits
//    clear, so e * hi is exact) and a low part;
//  * sin / cos from their Taylor series (to x^9 and x^10) on [-pi/4, pi/4]
//    after an exact reduction of the dyadic u2 to the nearest quarter turn.
//
// Every float operation is an explicit round-to-nearest intrinsic, so no
// multiply-add contraction can change a bit: the values are reproducible by
// any IEEE-754 single-precision implementation of the same steps.
#pragma once
#include <stdint.h>

namespace zo {

#define ZO_GAMMA 0x9E3779B97F4A7C15ull

__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Key of factor U (which = 0, keyed by the step) or V (which = 1, keyed by
// the first step of its lazy window).
__host__ __device__ __forceinline__ uint64_t factor_key(uint64_t run_seed, uint64_t step,
                                                       uint64_t nu, uint32_t layer,
                                                       uint32_t matrix, uint32_t which) {
    const uint64_t sp = which == 0 ? step : nu * (step / nu);
    uint64_t k = sm64_mix(run_seed);
    k = sm64_mix(k ^ sp);
    k = sm64_mix(k ^ (uint64_t)layer);
    return sm64_mix(k ^ (uint64_t)(matrix * 2u + which));
}

// Initial weights use a step value no direction reaches (all ones).
__host__ __device__ __forceinline__ uint64_t weight_key(uint64_t seed, uint32_t layer,
                                                       uint32_t tensor) {
    uint64_t k = sm64_mix(seed);
    k = sm64_mix(k ^ 0xFFFFFFFFFFFFFFFFull);
    k = sm64_mix(k ^ (uint64_t)layer);
    return sm64_mix(k ^ (uint64_t)tensor);
}

__device__ __forceinline__ float own_ln(float u) {
    // u in [2^-24, 1]: never subnormal, never zero
    const float kSqrt2 = static_cast<float>(1.4142135623730951);
    uint32_t bits = __float_as_uint(u);
    int e = (int)(bits >> 23) - 127;
    float m = __uint_as_float((bits & 0x7FFFFFu) | 0x3F800000u);
    if (m > kSqrt2) { m = __fmul_rn(m, 0.5f); e += 1; }
    const float s = __fdiv_rn(__fadd_rn(m, -1.0f), __fadd_rn(m, 1.0f));
    const float s2 = __fmul_rn(s, s);
    float p = static_cast<float>(1.0 / 11.0);
    p = __fadd_rn(__fmul_rn(p, s2), static_cast<float>(1.0 / 9.0));
    p = __fadd_rn(__fmul_rn(p, s2), static_cast<float>(1.0 / 7.0));
    p = __fadd_rn(__fmul_rn(p, s2), static_cast<float>(1.0 / 5.0));
    p = __fadd_rn(__fmul_rn(p, s2), static_cast<float>(1.0 / 3.0));
    p = __fadd_rn(__fmul_rn(p, s2), 1.0f);
    const float ln_m = __fmul_rn(__fmul_rn(s, p), 2.0f);
    // ln 2 = 0.6931471805599453 (double); float(ln 2) = 0x3F317218, high part 0x3F317200
    const float ln2_hi = __uint_as_float(0x3F317200u);
    const float ln2_lo = static_cast<float>(0.6931471805599453 - 0.693145751953125);
    const float ef = (float)e;
    return __fadd_rn(__fmul_rn(ef, ln2_hi), __fadd_rn(__fmul_rn(ef, ln2_lo), ln_m));
}

// sin and cos of 2 pi k / 2^24 for integer k in [0, 2^24).
__device__ __forceinline__ void own_sincos_turn(uint32_t k, float* sn, float* cs) {
    const int qn = (int)((k + (1u << 21)) >> 22);          // nearest quarter turn (0..4)
    const int q = qn & 3;
    const int fi = (int)k - (qn << 22);                       // [-2^21, 2^21]
    const float f = __fmul_rn((float)fi, 5.9604644775390625e-08f);   // * 2^-24, exact
    const float th = __fmul_rn(f, static_cast<float>(6.283185307179586));
    const float t2 = __fmul_rn(th, th);
    float ps = static_cast<float>(1.0 / 362880.0);
    ps = __fadd_rn(__fmul_rn(ps, t2), static_cast<float>(-1.0 / 5040.0));
    ps = __fadd_rn(__fmul_rn(ps, t2), static_cast<float>(1.0 / 120.0));
    ps = __fadd_rn(__fmul_rn(ps, t2), static_cast<float>(-1.0 / 6.0));
    const float s = __fadd_rn(th, __fmul_rn(__fmul_rn(th, t2), ps));
    float pc = static_cast<float>(-1.0 / 3628800.0);
    pc = __fadd_rn(__fmul_rn(pc, t2), static_cast<float>(1.0 / 40320.0));
    pc = __fadd_rn(__fmul_rn(pc, t2), static_cast<float>(-1.0 / 720.0));
    pc = __fadd_rn(__fmul_rn(pc, t2), static_cast<float>(1.0 / 24.0));
    pc = __fadd_rn(__fmul_rn(pc, t2), static_cast<float>(-1.0 / 2.0));
    const float c = __fadd_rn(1.0f, __fmul_rn(t2, pc));
    switch (q) {
        case 0: *sn = s;  *cs = c;  break;
        case 1: *sn = c;  *cs = -s; break;
        case 2: *sn = -s; *cs = -c; break;
        default: *sn = -c; *cs = s; break;
    }
}

// Pair j of the stream keyed by `key`: (z0, z1) = elements 2j and 2j+1.
__device__ __forceinline__ void normal_pair(uint64_t key, uint64_t j, float* z0, float* z1) {
    const uint64_t b = sm64_mix(key + (j + 1ull) * ZO_GAMMA);
    const float u1 = __fmul_rn((float)(uint32_t)((b >> 40) + 1ull), 5.9604644775390625e-08f);
    const float rho = __fsqrt_rn(__fmul_rn(-2.0f, own_ln(u1)));
    float sn, cs;
    own_sincos_turn((uint32_t)(b & 0xFFFFFFull), &sn, &cs);
    *z0 = __fmul_rn(rho, cs);
    *z1 = __fmul_rn(rho, sn);
}

}  // namespace zo
