// kda_tri.cuh -- the inverse of the 64 x 64 unit lower-triangular matrix I + N in
// fp32 on the CUDA cores, shared by the chunk-local forward and backward kernels
// (the UT/WY transform of a 64-token chunk needs (I + Diag(beta) A)^-1).
#pragma once
#include "kda_sm100.cuh"

namespace kda {

constexpr int TRI_LDA = 68;  // padded fp32 row stride of N and X (16-byte rows, spread banks)

// X = (I + N)^-1 for a strictly lower-triangular N [64][TRI_LDA] (fp32, shared memory),
// by the first 192 of the CTA's threads (every thread of the CTA must call it: it
// synchronises the CTA), blocked on 16x16 tiles: (1) the four diagonal blocks by forward
// substitution, (2) the sub-diagonal blocks of the two 32x32 diagonal halves,
// X_{b+1,b} = -X_{b+1,b+1} N_{b+1,b} X_bb (b = 0, 2), (3) the lower-left 32x32 block
// X_LL = -H_1 N_LL H_0 (H_0, H_1 the halves).  Blocks above the diagonal of X are never
// written or read.  sY: 8 KB of scratch.  sP [16][32] may overlay N (dead by then): it
// receives the second half of the sums of X's rows 48..63, columns 0..31, which the
// caller adds to those entries of X when it reads them.  Ends with a __syncthreads.
KDA_DEV void tri_inverse64(const float* sA, float* sX, float* sY, float* sP, int tid) {
    constexpr int LDA = TRI_LDA;
    if (tid < 64) {  // diagonal blocks: one thread per (block, column)
        // column j of (I + N_bb)^-1: x_i = -sum_{m<i} N_im x_m, x_j = 1, x_i = 0 for i < j
        // (entries above j are zero, so the sums need no masking)
        const int b = tid >> 4, j = tid & 15;
        const float* Nb = sA + (16 * b) * LDA + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float nr[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v4 = reinterpret_cast<const float4*>(Nb + i * LDA)[q];
                nr[4 * q] = v4.x; nr[4 * q + 1] = v4.y; nr[4 * q + 2] = v4.z; nr[4 * q + 3] = v4.w;
            }
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) {
                if (m & 1) acc1 += nr[m] * x[m];
                else acc0 += nr[m] * x[m];
            }
            x[i] = (i < j) ? 0.f : ((i == j) ? 1.f : -(acc0 + acc1));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sX[(16 * b + i) * LDA + 16 * b + j] = x[i];
    }
    __syncthreads();
    // Products below use 2x4 register tiles: acc[i][j] += sum_{m < 16} R[i][m] C[m][j]
    // (16-byte loads of 4 row entries and of 4 column entries feed 8 FMAs each);
    // a long sum is split over warp groups into partials that the next step adds.
    auto tile24 = [](const float* R, int ldr, const float* C, int ldc, float (&acc)[2][4]) {
#pragma unroll 2
        for (int m = 0; m < 16; m += 4) {
            float rv[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float4 v = *reinterpret_cast<const float4*>(R + i * ldr + m);
                rv[i][0] = v.x; rv[i][1] = v.y; rv[i][2] = v.z; rv[i][3] = v.w;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 cv = *reinterpret_cast<const float4*>(C + (m + k) * ldc);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    acc[i][0] += rv[i][k] * cv.x; acc[i][1] += rv[i][k] * cv.y;
                    acc[i][2] += rv[i][k] * cv.z; acc[i][3] += rv[i][k] * cv.w;
                }
            }
        }
    };
    auto store24 = [](float* D, int ldd, const float (&acc)[2][4], float sg) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
            *reinterpret_cast<float4*>(D + i * ldd) =
                make_float4(sg * acc[i][0], sg * acc[i][1], sg * acc[i][2], sg * acc[i][3]);
    };
    float* sZ0 = sY;          // [32][16] partial of Z over m in block 0 (columns of block 0)
    float* sZ1 = sY + 512;    // [32][32] partial of Z over m in block 1
    // (2a) Y_b = N_{b+1,b} X_bb  (b = 0, 2; 64 tiles, warps 0-1)
    if (tid < 64) {
        const int b = 2 * (tid >> 5), k = tid & 31, r0 = 2 * (k >> 2), c0 = 4 * (k & 3);
        float acc[2][4] = {};
        tile24(sA + (16 * (b + 1) + r0) * LDA + 16 * b, LDA, sX + (16 * b) * LDA + 16 * b + c0, LDA, acc);
        store24(sY + 1536 + (b >> 1) * 256 + r0 * 16 + c0, 16, acc, 1.f);
    }
    __syncthreads();
    // (2b) X_{b+1,b} = -X_{b+1,b+1} Y_b
    if (tid < 64) {
        const int b = 2 * (tid >> 5), k = tid & 31, r0 = 2 * (k >> 2), c0 = 4 * (k & 3);
        float acc[2][4] = {};
        tile24(sX + (16 * (b + 1) + r0) * LDA + 16 * (b + 1), LDA, sY + 1536 + (b >> 1) * 256 + c0, 16, acc);
        store24(sX + (16 * (b + 1) + r0) * LDA + 16 * b + c0, LDA, acc, -1.f);
    }
    __syncthreads();
    // (3a) Z = N_LL H_0 split over m: warps 0-1 m in block 0 (only the columns of block 0:
    //      H_0 is zero above its diagonal blocks), warps 2-5 m in block 1 (all columns)
    if (tid < 192) {
        const int g = tid >= 64;
        const int k = g ? tid - 64 : tid;
        const int r0 = g ? 2 * (k >> 3) : 2 * (k >> 2), c0 = g ? 4 * (k & 7) : 4 * (k & 3);
        float acc[2][4] = {};
        tile24(sA + (32 + r0) * LDA + 16 * g, LDA, sX + (16 * g) * LDA + c0, LDA, acc);
        if (g) store24(sZ1 + r0 * 32 + c0, 32, acc, 1.f);
        else store24(sZ0 + r0 * 16 + c0, 16, acc, 1.f);
    }
    __syncthreads();
    // Z = Z^(1) + Z^(0) on the columns of block 0 (32 x 16, one float4 per thread)
    if (tid < 128) {
        const int r = tid >> 2, c4 = 4 * (tid & 3);
        float4* z = reinterpret_cast<float4*>(sZ1 + r * 32 + c4);
        const float4 z0 = *reinterpret_cast<const float4*>(sZ0 + r * 16 + c4);
        float4 v = *z;
        v.x += z0.x; v.y += z0.y; v.z += z0.z; v.w += z0.w;
        *z = v;
    }
    __syncthreads();
    // (3b) X_LL = -H_1 Z (Z complete in sZ1) split over m: warps 0-3 m in block 2 (every row), warps 4-5 m in
    //      block 3 (rows of block 3 only), kept as a partial that the T image adds
    if (tid < 192) {
        const int g = tid >= 128;
        const int k = g ? tid - 128 : tid;
        const int r0 = g ? 16 + 2 * (k >> 3) : 2 * (k >> 3), c0 = 4 * (k & 7);
        float acc[2][4] = {};
        tile24(sX + (32 + r0) * LDA + 32 + 16 * g, LDA, sZ1 + (16 * g) * 32 + c0, 32, acc);
        if (g) store24(sP + (r0 - 16) * 32 + c0, 32, acc, -1.f);
        else store24(sX + (32 + r0) * LDA + c0, LDA, acc, -1.f);
    }
    __syncthreads();
}

}  // namespace kda
