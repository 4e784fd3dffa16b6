/*
 * Float64 CPU oracle of the TTT forward scan (TTT-Linear and TTT-MLP), from
 * "Learning to (Learn at Test Time): RNNs with Expressive Hidden States".
 *
 * TEST INFRASTRUCTURE.  Plain, slow, token-by-token loops that materialise the
 * per-token state W_t.  It shares no code with the CUDA library.  Only the
 * test suite, the smoke check and the bench's CPU-baseline leg may call it.
 *
 * The arithmetic lives in ttt_oracle_impl.h and is instantiated twice:
 *   oracle_*_f64 : REAL = double  -- the oracle
 *   oracle_*_f32 : REAL = float   -- the same loops in single precision, used
 *                                    only to measure rounding growth
 *
 * Parity pins (tests/test_oracle.py): Theorem 1 closed form, central finite
 * differences and autograd for every gradient, b = 1 against online GD,
 * eta = 0, state continuation, LayerNorm and GELU against library routines;
 * decode (linear and MLP) in pieces against the mini-batch rule written out
 * with autograd, and single-token plain decode against Theorem 1.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_MODE_LN_RESIDUAL 0
#define ORACLE_MODE_PLAIN 1

#define REAL double
#define SFX _f64
#define SQRT sqrt
#define TANH tanh
#include "ttt_oracle_impl.h"
#undef REAL
#undef SFX
#undef SQRT
#undef TANH

#define REAL float
#define SFX _f32
#define SQRT sqrtf
#define TANH tanhf
#include "ttt_oracle_impl.h"
#undef REAL
#undef SFX
#undef SQRT
#undef TANH
