// gdn_tc_inverse.cuh -- the blocked unit-lower-triangular inverse T = (I + A)^-1 of one chunk
// (64 x 64, A strictly lower), used by the WY kernel.
//
// A and T share one fp32 64 x 64 array X (row stride kXs floats): A is strictly lower and T
// unit lower-triangular, so A sits below the diagonal and T (off its unit diagonal) above it,
// transposed: X[r][s] = A[r][s] and X[s][r] = T[r][s] for r > s.  The four 16 x 16 diagonal
// blocks are solved by fp32 forward substitution (threads 0..63 of the 128 that run it), then
// three merge levels run as warp-level tf32 MMAs (four warps).  Every X entry that feeds a
// merge is stored already rounded to tf32 (round to nearest, ties away), so the merges issue no
// conversions; the diagonal blocks of A stay fp32 for the substitution.  Once solved, a diagonal
// block of X holds its block of T^T whole (the unit diagonal, and zeros where A was), so every
// read of a diagonal T block, here and in the caller, takes X as it stands.
#pragma once

#include <stdint.h>

namespace gdn {
namespace tc {

constexpr int kXs = 72;  // row stride (floats) of X: conflict-free 64-bit fragment reads

// fp32 -> tf32 (round to nearest, ties away), kept as an fp32 value whose low 13 mantissa bits
// are zero: mma.sync reads it as that tf32 value exactly.  The rounding is done on the bit
// pattern (sign-magnitude): adding half a tf32 unit (bit 12) to the magnitude and clearing the 13
// dropped bits rounds to nearest with ties away from zero, and a carry out of the mantissa steps
// the exponent as it should; two integer operations, no conversion unit.  Inputs are finite.  In
// the merges this rounding adds a relative error of about 1e-6 to T (|T - T_exact| / |T| over
// random chunks of the workloads' distributions), some thirty times below the bf16 rounding that
// the T image gets afterwards.
__device__ __forceinline__ float tf32r(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// D += A B for one 16 x 8 x 8 tile in tf32 (A row-major, B column-major, D fp32); the operands
// are tf32 values held in fp32 registers
__device__ __forceinline__ void mma_tf32(float* d, float a0, float a1, float a2, float a3, float b0,
                                         float b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(__float_as_uint(a0)), "r"(__float_as_uint(a1)), "r"(__float_as_uint(a2)),
          "r"(__float_as_uint(a3)), "r"(__float_as_uint(b0)), "r"(__float_as_uint(b1)));
}

// The four 16 x 16 diagonal blocks of T (threads 0..63: block t / 16, column t % 16): unit
// lower-triangular inverse by forward substitution, reading each A row as 16-byte vectors.
// Column cc of block b is T[16 b + r][16 b + cc] = x[r] (x[r] = 0 for r < cc, x[cc] = 1); it is
// written whole to row 16 b + cc of X once every thread has read its A block (the caller's
// barrier sits in between).
__device__ __forceinline__ void diag_solve(const float* X, int t, float* x) {
    const int b = t >> 4, cc = t & 15;
    const float* a = X + 16 * b * (kXs + 1);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        float row[16];
#pragma unroll
        for (int q = 0; q < (r + 3) / 4; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(a + r * kXs + 4 * q);
            row[4 * q] = v.x;
            row[4 * q + 1] = v.y;
            row[4 * q + 2] = v.z;
            row[4 * q + 3] = v.w;
        }
        float s0 = (r == cc) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j + 1 < r; j += 2) {
            s0 -= row[j] * x[j];
            s1 -= row[j + 1] * x[j + 1];
        }
        if (r & 1) s0 -= row[r - 1] * x[r - 1];
        x[r] = (r < cc) ? 0.f : s0 + s1;
    }
}

__device__ __forceinline__ void diag_store(float* X, int t, const float* x) {
    const int b = t >> 4, cc = t & 15;
    float* m = X + (16 * b + cc) * kXs + 16 * b;  // entries left of the diagonal are no longer read
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(m + 4 * q) =
            make_float4(tf32r(x[4 * q]), tf32r(x[4 * q + 1]), tf32r(x[4 * q + 2]), tf32r(x[4 * q + 3]));
}

// Level D (1..3) of the blocked inverse on the tensor cores: for the blocks (i, j0 = i - D),
//   Y = sum_{k = j0}^{i-1} A_ik T_k,j0,   T_i,j0 = -T_ii Y      (16 x 16 blocks)
// A work unit is one 8-column half of one block (one m16n8 tile); warp w takes units w, w + 4.
// In Y the k slots (t, t + 4) of lane (g, t) stand for the adjacent columns (2t, 2t + 1), so
// that A and T come in as 64-bit pairs; in T_ii Y the M slots (g, g + 8) stand for the adjacent
// rows (2g, 2g + 1), which makes both the T_ii fragment and the result 64-bit pairs in X.
// Y goes from the accumulator layout to the B-operand layout through a per-warp 16 x 9 scratch.
template <int D>
__device__ __forceinline__ void merge_level(float* X, float* ysw, int warp, int lane) {
    constexpr int kUnits = 2 * (4 - D);
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int u = warp; u < kUnits; u += 4) {
        const int i = D + (u >> 1), j0 = i - D, col = 16 * j0 + 8 * (u & 1);
        const int r0 = 16 * i + g;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kb = 0; kb < D; ++kb) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int kc = 16 * (j0 + kb) + 8 * ks + 2 * t;
                const float2 a0 = *reinterpret_cast<const float2*>(X + r0 * kXs + kc);
                const float2 a1 = *reinterpret_cast<const float2*>(X + (r0 + 8) * kXs + kc);
                const float2 bv = *reinterpret_cast<const float2*>(X + (col + g) * kXs + kc);
                mma_tf32(y, a0.x, a1.x, a0.y, a1.y, bv.x, bv.y);
            }
        }
        ysw[g * 9 + 2 * t] = tf32r(y[0]);
        ysw[g * 9 + 2 * t + 1] = tf32r(y[1]);
        ysw[(g + 8) * 9 + 2 * t] = tf32r(y[2]);
        ysw[(g + 8) * 9 + 2 * t + 1] = tf32r(y[3]);
        __syncwarp();
        const int rr = 16 * i + 2 * g;  // rows rr, rr + 1 of T_ii
        float r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int kc = 16 * i + 8 * ks + t;
            const float2 p0 = *reinterpret_cast<const float2*>(X + kc * kXs + rr);
            const float2 p1 = *reinterpret_cast<const float2*>(X + (kc + 4) * kXs + rr);
            mma_tf32(r, p0.x, p0.y, p1.x, p1.y, ysw[(8 * ks + t) * 9 + g], ysw[(8 * ks + t + 4) * 9 + g]);
        }
        __syncwarp();  // the scratch is rewritten by this warp's next unit
        // T block (i, j0), transposed into X above the diagonal
        *reinterpret_cast<float2*>(X + (col + 2 * t) * kXs + rr) = make_float2(tf32r(-r[0]), tf32r(-r[2]));
        *reinterpret_cast<float2*>(X + (col + 2 * t + 1) * kXs + rr) = make_float2(tf32r(-r[1]), tf32r(-r[3]));
    }
}

}  // namespace tc
}  // namespace gdn
