/*
 * moe_oracle_f32.c -- the CPU oracle of moe_oracle.c compiled with single
 * precision arithmetic, for TIMING ONLY.
 *
 * TEST INFRASTRUCTURE ONLY.  The bench's CPU-baseline leg times this build
 * beside the fp64 oracle (the fp64 build, moe_oracle.c alone, is the one the
 * tests check against; this build is never used as a reference).  Every
 * `double` of moe_oracle.c becomes `float` here: values, accumulators and the
 * exported functions' floating-point arguments, so the loops run as a plain
 * fp32 CPU implementation of the same definition, in the same order.
 * Library calls (exp, tanh, sqrt, ldexp) keep their double prototypes from
 * the headers included first; their results are rounded to float on
 * assignment.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define double float
#include "moe_oracle.c"
