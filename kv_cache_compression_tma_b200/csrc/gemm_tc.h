// gemm_tc.h -- split-tf32 tensor-core GEMM for the absorb (see gemm_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ispa {

// Two tensor maps over one row-major fp32 matrix: K-major tiles {32 cols, 128 rows} and MN-major
// tiles {32 cols, 32 rows}, both with 128-byte swizzle.
struct F32Operand {
  const float* base;
  CUtensorMap kmajor;
  CUtensorMap mnmajor;
};

bool make_operand_maps(F32Operand* op, const float* base, uint64_t rows, uint64_t cols, uint64_t ld);
bool make_map_f32_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                     uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// C = alpha * op(A) op(B) (accumulate = false) or C += alpha * op(A) op(B) (accumulate = true), where
// op(A)'s storage starts at (a_r0, a_c0) of A's matrix, op(B)'s at (b_r0, b_c0) of B's and C's block at
// (c_r0, c_c0) of C's.  M, N multiples of 128, K a multiple of 32.  C may alias A's block when N == 128,
// or B's block when M == 128 (each CTA reads its whole input panel before its stores are issued).
// pdl: launch with programmatic stream serialisation (the kernel's prologue overlaps the previous
// grid of the stream; its first access to operands waits for that grid to complete).
// exact: bit 0 = every value of A is a tf32 number (a widened bf16 matrix), bit 1 = the same for B;
// an exact operand's lo part is zero, so its split and the products with its lo part are skipped
// (hi*hi + lo*hi for an exact B, hi*hi alone when both are exact).
cudaError_t gemm_tc(bool ta, bool tb, int M, int N, int K, float alpha, const F32Operand& A, int a_r0, int a_c0,
                    const F32Operand& B, int b_r0, int b_c0, bool accumulate, const F32Operand& C, int c_r0, int c_c0,
                    bool lower_only, unsigned* status, cudaStream_t s, int* n_launched, bool pdl = false,
                    int exact = 0);

}  // namespace ispa
