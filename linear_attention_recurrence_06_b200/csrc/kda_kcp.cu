// kda_kcp.cu -- the fold step of context parallelism across devices.
//
// A sequence cut into consecutive segments (one per device) is linear in its
// initial state: segment r maps S -> M_r S + B_r (M_r: dk x dk, B_r: dk x dv),
// and the initial state of segment r is the composition of the maps of
// segments 0 .. r-1 applied to the sequence's initial state ("training and
// inference systems" item of the K3 article summaries, xhh.club tag page:
// context parallelism as a prefix scan of segment transitions; the nlpx.cn K3
// walkthrough, §6: KCP).  After the maps are gathered from every device, each
// device folds the ones before it:
//     S <- S_0;  for j = 0 .. n_prev-1:  S <- M_j S + B_j.
// n_prev <= world size - 1 small dense products per head: fp32 FMA on the
// CUDA cores, no tensor cores (a few microseconds at 8 devices and 32 heads).
#include "kda_launch.h"
#include "kda_profile.h"

namespace kda {
namespace {

constexpr int D = 128;        // dk = dv
constexpr int CS = 32;        // state columns per CTA
constexpr int CP_THREADS = 256;

// gathered maps: trans[r][0][n][h] = M_r (dk x dk), trans[r][1][n][h] = B_r (dk x dv), fp32 row-major.
// One CTA = columns [32 js, 32 js + 32) of one (sequence, head) state.  Thread t
// owns rows 4 (t / 8) .. + 4 and columns 4 (t % 8) .. + 4 of that slice: per key
// index k one 16-byte shared load of S[k] feeds 16 FMAs, and the four M rows
// stream from global memory (L1-resident across the 8 threads that share them).
__global__ void __launch_bounds__(CP_THREADS)
kcp_compose_kernel(const float* __restrict__ trans, int n_prev, const float* __restrict__ init_state,
                   float* __restrict__ state_in, int N, int H) {
    __shared__ float4 sS[2][D][CS / 4];  // ping-pong state slices, 2 x 16 KB
    const int js = blockIdx.x, h = blockIdx.y, n = blockIdx.z, t = threadIdx.x;
    const size_t mat = ((size_t)n * H + h) * D * D;
    const size_t half = (size_t)N * H * D * D;  // elements of all M (or all B) of one device
    const int col0 = CS * js;
    for (int e = t; e < D * CS / 4; e += CP_THREADS) {
        const int r = e / (CS / 4), c4 = e % (CS / 4);
        sS[0][r][c4] = init_state ? *reinterpret_cast<const float4*>(init_state + mat + (size_t)r * D + col0 + 4 * c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const int i0 = 4 * (t >> 3), cq = t & 7;
    int cur = 0;
    for (int j = 0; j < n_prev; ++j) {
        const float* M = trans + (size_t)j * 2 * half + mat;
        const float* Bj = M + half;
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float4 b = *reinterpret_cast<const float4*>(Bj + (size_t)(i0 + r) * D + col0 + 4 * cq);
            acc[r][0] = b.x; acc[r][1] = b.y; acc[r][2] = b.z; acc[r][3] = b.w;
        }
#pragma unroll 2
        for (int kk = 0; kk < D / 4; ++kk) {
            float m[4][4];  // M[i0 + r][4 kk + u]
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float4 v = *reinterpret_cast<const float4*>(M + (size_t)(i0 + r) * D + 4 * kk);
                m[r][0] = v.x; m[r][1] = v.y; m[r][2] = v.z; m[r][3] = v.w;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 s = sS[cur][4 * kk + u][cq];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    acc[r][0] = fmaf(m[r][u], s.x, acc[r][0]);
                    acc[r][1] = fmaf(m[r][u], s.y, acc[r][1]);
                    acc[r][2] = fmaf(m[r][u], s.z, acc[r][2]);
                    acc[r][3] = fmaf(m[r][u], s.w, acc[r][3]);
                }
            }
        }
        // the other buffer was last read before the previous step's barrier
#pragma unroll
        for (int r = 0; r < 4; ++r) sS[cur ^ 1][i0 + r][cq] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        __syncthreads();
        cur ^= 1;
    }
    for (int e = t; e < D * CS / 4; e += CP_THREADS) {
        const int r = e / (CS / 4), c4 = e % (CS / 4);
        *reinterpret_cast<float4*>(state_in + mat + (size_t)r * D + col0 + 4 * c4) = sS[cur][r][c4];
    }
}

}  // namespace

cudaError_t launch_kcp_compose(const float* trans, int n_prev, const float* init_state, float* state_in, int N, int H,
                               cudaStream_t stream) {
    if (N == 0) return cudaSuccess;
    prof_begin(PROF_KCP_COMPOSE, stream);
    kcp_compose_kernel<<<dim3(D / CS, H, N), CP_THREADS, 0, stream>>>(trans, n_prev, init_state, state_in, N, H);
    const cudaError_t err = cudaGetLastError();
    prof_end(PROF_KCP_COMPOSE, stream);
    return err;
}

}  // namespace kda
