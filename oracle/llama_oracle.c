/*
 * CPU oracle of one Llama-style decode step.  TEST INFRASTRUCTURE ONLY: only
 * the tests, the package smoke check and the bench's CPU-baseline leg may
 * load it.  It shares no code with the GPU engine.
 *
 * The body is included twice: double precision (the definition, suffix _f64)
 * and single precision with sequential accumulation (suffix _f32).
 */
#include "llama_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define R double
#define S _f64
#include "llama_oracle_body.h"
#undef R
#undef S

#define R float
#define S _f32
#include "llama_oracle_body.h"
#undef R
#undef S

int orc_argmax(const double *x, int n) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (x[i] > x[best]) best = i;
  return best;
}
