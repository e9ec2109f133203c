// slay_exp2_poly.h -- written by gen_exp2_poly.py; do not edit.
// 2^f ~= c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2], minimax in relative error;
// largest relative error of the float32 Horner evaluation: 7.485e-05
#pragma once

#define SLAY_EXP2_C0 9.999280572e-01f
#define SLAY_EXP2_C1 6.932608485e-01f
#define SLAY_EXP2_C2 2.426111549e-01f
#define SLAY_EXP2_C3 5.517221987e-02f
#define SLAY_EXP2_MAX_REL_ERR 7.485e-05
