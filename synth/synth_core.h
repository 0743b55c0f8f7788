/*
 * synth_core.h -- the seeded synthetic-input generator shared by the CPU
 * oracle side and the GPU side.  It holds none of the MoE / FP4 arithmetic:
 * it only turns (seed, stream, index) into numbers.
 *
 * Definition (the same on host and device, bit for bit):
 *
 *   mix(z)      : the splitmix64 output function (Steele, Lea, Flood,
 *                 "Fast splittable pseudorandom number generators", 2014):
 *                 z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                 z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31.
 *   key(s, t)   = mix(s * G + mix(t + 1)),          G = 0x9E3779B97F4A7C15
 *   u64(s,t,i)  = mix(key(s,t) + (i + 1) * G)       (splitmix64 evaluated at
 *                                                    counter i, so any index
 *                                                    can be drawn directly)
 *   normal pair j (Box-Muller, Box & Muller 1958), a = u64(2j), b = u64(2j+1):
 *       u1 = ((a >> 11) + 1) * 2^-53   in (0, 1]
 *       u2 =  (b >> 11)      * 2^-53   in [0, 1)
 *       r  = sqrt(-2 ln u1),  z_{2j} = r cos(2 pi u2),  z_{2j+1} = r sin(2 pi u2)
 *
 * ln, cos and sin are evaluated here with IEEE double +, -, *, / and sqrt
 * only (all correctly rounded on both CPU and GPU) and no fused multiply-add,
 * so the host and the device produce identical doubles:
 *   ln(m 2^e) = e ln2 + 2 atanh((m-1)/(m+1)),  m in [sqrt(1/2), sqrt(2)),
 *               atanh by its odd power series (11 terms; |s| <= 0.1716);
 *   cos, sin of phi = f pi/2, f in [0,1), by their Taylor series to x^22 /
 *               x^23, then rotated by the exact quadrant of u2.
 * Rounding to fp32 is one double->float round-to-nearest-even; bf16 is the
 * round-to-nearest-even of that fp32 value.
 *
 * The including file defines SYNTH_FN (function qualifiers) and the four
 * double operations SYNTH_ADD/SUB/MUL/DIV and SYNTH_SQRT before including.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

SYNTH_FN uint64_t synth_mix64(uint64_t z)
{
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t stream)
{
    return synth_mix64(seed * SYNTH_GOLDEN + synth_mix64(stream + 1));
}

SYNTH_FN uint64_t synth_u64_k(uint64_t key, uint64_t i)
{
    return synth_mix64(key + (i + 1) * SYNTH_GOLDEN);
}

SYNTH_FN double synth_bits_to_double(uint64_t b)
{
    union { uint64_t u; double d; } c;
    c.u = b;
    return c.d;
}

SYNTH_FN uint64_t synth_double_to_bits(double d)
{
    union { uint64_t u; double d; } c;
    c.d = d;
    return c.u;
}

/* natural log of u in (0, 1] (u is a normal double) */
SYNTH_FN double synth_ln(double u)
{
    uint64_t bits = synth_double_to_bits(u);
    int e = (int)((bits >> 52) & 0x7FF) - 1023;
    double m = synth_bits_to_double((bits & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL);
    if (m > 1.4142135623730951) {                 /* m in (sqrt2, 2) -> halve */
        m = synth_bits_to_double((bits & 0x000FFFFFFFFFFFFFULL) | 0x3FE0000000000000ULL);
        e += 1;
    }
    double s = SYNTH_DIV(SYNTH_SUB(m, 1.0), SYNTH_ADD(m, 1.0));
    double s2 = SYNTH_MUL(s, s);
    double p = 1.0 / 21.0;
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 19.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 17.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 15.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 13.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 11.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 9.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 7.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 5.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0 / 3.0);
    p = SYNTH_ADD(SYNTH_MUL(p, s2), 1.0);
    double lnm = SYNTH_MUL(SYNTH_MUL(2.0, s), p);
    return SYNTH_ADD(SYNTH_MUL((double)e, 0.6931471805599453), lnm);
}

/* cos and sin of phi in [0, pi/2) by Taylor series */
SYNTH_FN void synth_cossin_q(double phi, double* c, double* s)
{
    double x2 = SYNTH_MUL(phi, phi);
    /* cos: sum_{n=0..11} (-1)^n x^{2n} / (2n)! , Horner in x2 */
    double pc = 1.0 / 1124000727777607680000.0;         /* 1/22! */
    pc = SYNTH_SUB(1.0 / 2432902008176640000.0, SYNTH_MUL(pc, x2)); /* 1/20! */
    pc = SYNTH_SUB(1.0 / 6402373705728000.0, SYNTH_MUL(pc, x2));    /* 1/18! */
    pc = SYNTH_SUB(1.0 / 20922789888000.0, SYNTH_MUL(pc, x2));      /* 1/16! */
    pc = SYNTH_SUB(1.0 / 87178291200.0, SYNTH_MUL(pc, x2));         /* 1/14! */
    pc = SYNTH_SUB(1.0 / 479001600.0, SYNTH_MUL(pc, x2));           /* 1/12! */
    pc = SYNTH_SUB(1.0 / 3628800.0, SYNTH_MUL(pc, x2));             /* 1/10! */
    pc = SYNTH_SUB(1.0 / 40320.0, SYNTH_MUL(pc, x2));               /* 1/8!  */
    pc = SYNTH_SUB(1.0 / 720.0, SYNTH_MUL(pc, x2));                 /* 1/6!  */
    pc = SYNTH_SUB(1.0 / 24.0, SYNTH_MUL(pc, x2));                  /* 1/4!  */
    pc = SYNTH_SUB(1.0 / 2.0, SYNTH_MUL(pc, x2));                   /* 1/2!  */
    pc = SYNTH_SUB(1.0, SYNTH_MUL(pc, x2));
    /* sin: x * sum_{n=0..11} (-1)^n x^{2n} / (2n+1)! */
    double ps = 1.0 / 25852016738884976640000.0;        /* 1/23! */
    ps = SYNTH_SUB(1.0 / 51090942171709440000.0, SYNTH_MUL(ps, x2));   /* 1/21! */
    ps = SYNTH_SUB(1.0 / 121645100408832000.0, SYNTH_MUL(ps, x2));  /* 1/19! */
    ps = SYNTH_SUB(1.0 / 355687428096000.0, SYNTH_MUL(ps, x2));     /* 1/17! */
    ps = SYNTH_SUB(1.0 / 1307674368000.0, SYNTH_MUL(ps, x2));       /* 1/15! */
    ps = SYNTH_SUB(1.0 / 6227020800.0, SYNTH_MUL(ps, x2));          /* 1/13! */
    ps = SYNTH_SUB(1.0 / 39916800.0, SYNTH_MUL(ps, x2));            /* 1/11! */
    ps = SYNTH_SUB(1.0 / 362880.0, SYNTH_MUL(ps, x2));              /* 1/9!  */
    ps = SYNTH_SUB(1.0 / 5040.0, SYNTH_MUL(ps, x2));                /* 1/7!  */
    ps = SYNTH_SUB(1.0 / 120.0, SYNTH_MUL(ps, x2));                 /* 1/5!  */
    ps = SYNTH_SUB(1.0 / 6.0, SYNTH_MUL(ps, x2));                   /* 1/3!  */
    ps = SYNTH_SUB(1.0, SYNTH_MUL(ps, x2));
    *c = pc;
    *s = SYNTH_MUL(phi, ps);
}

/* standard normal number `i` of stream (seed, stream); key = synth_key(seed, stream) */
SYNTH_FN double synth_normal_k(uint64_t key, uint64_t i)
{
    uint64_t j = i >> 1;
    uint64_t a = synth_u64_k(key, 2 * j);
    uint64_t b = synth_u64_k(key, 2 * j + 1);
    double u1 = SYNTH_MUL((double)((a >> 11) + 1), 1.0 / 9007199254740992.0);
    uint64_t b53 = b >> 11;
    /* quadrant and fraction of u2 = b53 * 2^-53, both exact */
    uint32_t q = (uint32_t)(b53 >> 51);
    double f = SYNTH_MUL((double)(b53 & ((1ULL << 51) - 1)), 1.0 / 2251799813685248.0);
    double phi = SYNTH_MUL(f, 1.5707963267948966);
    double c, s;
    synth_cossin_q(phi, &c, &s);
    double cq, sq;
    switch (q) {
    case 0: cq = c;  sq = s;  break;
    case 1: cq = -s; sq = c;  break;
    case 2: cq = -c; sq = -s; break;
    default: cq = s; sq = -c; break;
    }
    double r = SYNTH_SQRT(SYNTH_MUL(-2.0, synth_ln(u1)));
    return SYNTH_MUL(r, (i & 1) ? sq : cq);
}

/* fp32 bits -> bf16 bits, round to nearest even (finite inputs only) */
SYNTH_FN uint16_t synth_f32_to_bf16_bits(uint32_t f)
{
    uint32_t lsb = (f >> 16) & 1u;
    return (uint16_t)((f + 0x7FFFu + lsb) >> 16);
}

#endif /* SYNTH_CORE_H */
