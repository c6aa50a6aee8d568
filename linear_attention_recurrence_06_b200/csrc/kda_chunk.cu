// kda_chunk.cu -- chunkwise prefill of the KDA recurrence on sm_100a.
//
// Source: K3 article summaries (xhh.club tag page), item "chunkwise parallel
// algorithm": the sequence is cut into chunks, the state recurs between
// chunks and matrix products run inside a chunk; the per-step log-decay has a
// lower bound of -5 so that 16-token diagonal tiles can use BF16 matrix
// multiplies.  Section 6 of the nlpx.cn K3 walkthrough adds the reason: the
// reciprocal of the cumulative decay overflows.
//
// Algebra for one chunk of C = 64 tokens of one head, starting from S0
// (g_t = in-chunk cumulative clamped log-decay, a dk-vector; Gam_t = e^{g_t}):
//   A[t][s] = sum_c k_tc k_sc e^{g_tc - g_sc}   (s < t)
//   P[t][s] = scale * sum_c q_tc k_sc e^{g_tc - g_sc}   (s <= t)
//   T  = (I + Diag(beta) A)^-1 Diag(beta)
//   W  = T (K o Gam),   Ut = T V,   Kt = K o e^{g_C - g}
// and the chunk acts on the state as an affine map (a segment transition, the
// object context parallelism composes by a prefix scan per the "training and
// inference systems" item):
//   S_C = Diag(Gam_C) S0 - Mlr S0 + Bm,       Mlr = Kt^T W,  Bm = Kt^T Ut
//   O   = Qp S0 + Ob,                          Qp = scale (Q o Gam) - P W,  Ob = P Ut
//
// Two kernels:
//   intra_kernel  one CTA per (chunk, head), all chunks in parallel.  Builds
//                 the decay-scaled operands, runs every product above on the
//                 tensor cores (tcgen05.mma, TMEM accumulators), inverts the
//                 64x64 unit-triangular system in fp32, and writes Mlr, Qp,
//                 Bm, Ob and Gam_C to the workspace.
//   chain_kernel  one CTA per (sequence, head, 32-column slice of dv); walks
//                 the chunks in order.  Per chunk ONE round of tensor-core
//                 products (Mlr S and Qp S, the state slice as the shared B
//                 operand), then S <- Gam_C o S - Mlr S + Bm in fp32 registers
//                 and o = Qp S + Ob.  Mlr/Qp tiles arrive by bulk copies
//                 (TMA engine), double-buffered one chunk ahead.
//
// Exponent references (why the -5 bound matters): inside a 64-token chunk the
// cumulative decay can reach e^{-320}, whose reciprocal overflows fp32/bf16.
// Each 16-token tile b uses its own reference G_b = g at the token before the
// tile (G_0 = 0).  Row operands carry e^{g_t - G_b} <= 1; column operands of
// the diagonal tile carry e^{G_b - g_s} <= e^{16*5} = e^80 (finite in bf16);
// column operands of earlier tiles carry e^{G_b - g_s} = e^{G_b - G_{bs+1}}
// e^{G_{bs+1} - g_s}, a product of two factors <= 1.  Every bf16 operand is
// finite and every product is a correctly-scaled e^{g_t - g_s}.
#include "kda_profile.h"
#include "kda_sm100.cuh"

namespace kda {

constexpr int CH = 64;    // chunk length
constexpr int DK = 128;   // key head dim
constexpr int DV = 128;   // value head dim
constexpr int DVS = 32;   // value columns per chain CTA

// Workspace bytes per (chunk, head) slot.
constexpr size_t SLOT_M = (size_t)DK * DK * 2;   // Mlr, bf16 K-major SW128 image [128][128]
constexpr size_t SLOT_Q = (size_t)CH * DK * 2;   // Qp,  bf16 K-major SW128 image [64][128]
constexpr size_t SLOT_B = (size_t)DK * DV * 2;   // Bm,  bf16 row-major [128][128]
constexpr size_t SLOT_O = (size_t)CH * DV * 2;   // Ob,  bf16 row-major [64][128]
constexpr size_t SLOT_G = (size_t)DK * 4;        // Gam_C, fp32 [128]

struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* log_alpha;
    const void* beta;
    const float* init_state;   // nullable
    float* state_io;           // carry / final state [N, H, dk, dv]
    void* o;
    const int32_t* cu;         // nullable (fixed length)
    uint8_t* ws_M;
    uint8_t* ws_Q;
    uint8_t* ws_B;
    uint8_t* ws_O;
    float* ws_G;
    uint32_t* status;
    int64_t T;                 // tokens per sequence (fixed) or total tokens (varlen)
    int H;
    int n_seqs;
    int i0;                    // first chunk index of this pass (within each sequence)
    int wc;                    // chunk slots per sequence in this pass
    int first_pass;
    float scale;
};

// Token range [sb, se) of sequence n, clamped into [0, total tokens].
KDA_DEV void seq_range(const ChunkArgs& a, int n, int64_t& sb, int64_t& se) {
    if (a.cu == nullptr) {
        sb = (int64_t)n * a.T;
        se = sb + a.T;
    } else {
        int64_t b = __ldg(a.cu + n), e = __ldg(a.cu + n + 1);
        b = b < 0 ? 0 : (b > a.T ? a.T : b);
        e = e < b ? b : (e > a.T ? a.T : e);
        sb = b;
        se = e;
    }
}

// Issues D (+)= A B^T over K (multiple of 16) for two K-major SW128 images.
// a_rows / b_rows are the row counts of one 128-byte-wide K block of each.
KDA_DEV void mma_run(uint32_t d, uint32_t a_addr, uint32_t a_rows, uint32_t b_addr, uint32_t b_rows, int K,
                     uint32_t idesc) {
    for (int kk = 0; kk < K / 16; ++kk) {
        const uint32_t kb = (uint32_t)kk >> 2, ks = (uint32_t)kk & 3u;
        const uint64_t ad = sdesc_k_sw128(a_addr + kb * a_rows * 128u + ks * 32u);
        const uint64_t bd = sdesc_k_sw128(b_addr + kb * b_rows * 128u + ks * 32u);
        mma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
}

// ---------------------------------------------------------------------------
// intra_kernel
// ---------------------------------------------------------------------------
// Threads: 256.  Thread tid owns key/value channel c = tid & 127 and tokens
// [32*half, 32*half + 32), half = tid >> 7.  Warp w reads TMEM lanes
// 32*(w & 3) .. +31, i.e. rows c = tid & 127, and its half selects columns.
//
// Shared memory (offsets from a 1024-aligned base):
//   X [0, 72K)      phase 1: KQr [128][128] @0, Kd [64][128] @32K,
//                            Kb1 [16][128] @48K, Kb2 [32][128] @52K, Kb3 [48][128] @60K
//                   phase 2: KGt [128][64] @0, Vt [128][64] @16K, Ti [64][64] @32K,
//                            Ktt [128][64] @40K, Ph [64][64] @56K, inverse temp @64K
//   Y [72K, 104K)   A fp32 [64][64] @0, X fp32 [64][64] @16K; later Wt [128][64] @0,
//                   Ut [128][64] @16K
//   misc            beta[64], G[5][128], half-0 totals[128], mbarrier, TMEM base
constexpr uint32_t IX_KQR = 0, IX_KD = 32768, IX_KB1 = 49152, IX_KB2 = 53248, IX_KB3 = 61440;
constexpr uint32_t IX_KGT = 0, IX_VT = 16384, IX_TI = 32768, IX_KTT = 40960, IX_PH = 57344, IX_TMP = 65536;
constexpr uint32_t IY = 73728;
constexpr uint32_t IY_A = IY, IY_X = IY + 16384, IY_WT = IY, IY_UT = IY + 16384;
constexpr uint32_t IM = IY + 32768;
constexpr uint32_t IM_BETA = IM, IM_G = IM + 256, IM_TOT = IM + 256 + 2560, IM_BAR = IM_TOT + 512,
                   IM_TMEM = IM_BAR + 8;
constexpr uint32_t INTRA_SMEM = IM_TMEM + 8 + 1024;  // + alignment slack
constexpr uint32_t INTRA_TMEM_COLS = 256;

template <bool IN_BF16>
__global__ void __launch_bounds__(256, 2) intra_kernel(const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = tid & 127, half = tid >> 7;
    const int qd = warp & 3;
    const int H = a.H, h = blockIdx.y;
    const int n = blockIdx.x / a.wc, ci = a.i0 + blockIdx.x % a.wc;
    int64_t s_beg, s_end;
    seq_range(a, n, s_beg, s_end);
    const int64_t t0 = s_beg + (int64_t)ci * CH;
    if (t0 >= s_end) return;  // chunk beyond this sequence: nothing to do
    const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
    const size_t slot = ((size_t)n * a.wc + (blockIdx.x % a.wc)) * H + h;

    float* s_beta = reinterpret_cast<float*>(sm + IM_BETA);
    float* s_G = reinterpret_cast<float*>(sm + IM_G);      // [5][128]
    float* s_tot = reinterpret_cast<float*>(sm + IM_TOT);  // [128]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + IM_BAR);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + IM_TMEM);

    if (warp == 0) {
        tmem_alloc(s_tmem, INTRA_TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (tid < CH) s_beta[tid] = (tid < L) ? ld_in<IN_BF16>(a.beta, (size_t)(t0 + tid) * H + h) : 0.f;

    // ---- phase 1: cumulative clamped log-decay g (registers), tile references G
    const size_t rowstride = (size_t)H * DK;
    const size_t ebase = ((size_t)t0 * H + h) * DK + c;  // element (t0, h, c)
    float gl[32];
    {
        float run = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int t = 32 * half + u;
            const float l = (t < L) ? fmaxf(ld_in<IN_BF16>(a.log_alpha, ebase + (size_t)t * rowstride),
                                            LOG_ALPHA_FLOOR)
                                    : 0.f;
            run += l;
            gl[u] = run;
        }
        if (half == 0) s_tot[c] = run;
    }
    __syncthreads();
    if (half == 1) {
        const float off = s_tot[c];
#pragma unroll
        for (int u = 0; u < 32; ++u) gl[u] += off;
    }
    // G_0 = 0, G_1 = g_15, G_2 = g_31, G_3 = g_47, G_4 = g_63 (= g at the chunk end)
    if (half == 0) {
        s_G[0 * 128 + c] = 0.f;
        s_G[1 * 128 + c] = gl[15];
        s_G[2 * 128 + c] = gl[31];
    } else {
        s_G[3 * 128 + c] = gl[15];
        s_G[4 * 128 + c] = gl[31];
    }
    __syncthreads();
    float G[5];
#pragma unroll
    for (int b = 0; b < 5; ++b) G[b] = s_G[b * 128 + c];

    // E1 = e^{g_t - G_bt} (<= 1),  E3 = e^{G_{bt+1} - g_t} (<= 1)
    float E1[32], E3[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
        const int bt = (32 * half + u) >> 4;  // compile-time per half after unrolling
        const float Gb = (bt == 0) ? G[0] : (bt == 1) ? G[1] : (bt == 2) ? G[2] : G[3];
        const float Gn = (bt == 0) ? G[1] : (bt == 1) ? G[2] : (bt == 2) ? G[3] : G[4];
        E1[u] = __expf(gl[u] - Gb);
        E3[u] = __expf(Gn - gl[u]);
    }

    // ---- phase 1 operands: KQr = [K o E1 ; scale Q o E1], Kd = K o e^{G_bt - g}, Kb^(b)
    {
        const uint32_t kb = (uint32_t)c >> 6, kc = (uint32_t)c & 63u;
        // factors e^{G_b - G_{bs+1}} for the off-diagonal column operands
        const float f21 = __expf(G[2] - G[1]), f31 = __expf(G[3] - G[1]), f32 = __expf(G[3] - G[2]);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int t = 32 * half + u;
            const int bt = t >> 4;
            const float kv = (t < L) ? ld_in<IN_BF16>(a.k, ebase + (size_t)t * rowstride) : 0.f;
            const float qv = (t < L) ? ld_in<IN_BF16>(a.q, ebase + (size_t)t * rowstride) : 0.f;
            const float kr = kv * E1[u];
            *reinterpret_cast<uint16_t*>(sm + IX_KQR + kb * 16384u + sw128_off(t, kc)) = f32_to_bf16(kr);
            *reinterpret_cast<uint16_t*>(sm + IX_KQR + kb * 16384u + sw128_off(t + 64, kc)) =
                f32_to_bf16(qv * E1[u] * a.scale);
            const float Gb = (bt == 0) ? G[0] : (bt == 1) ? G[1] : (bt == 2) ? G[2] : G[3];
            *reinterpret_cast<uint16_t*>(sm + IX_KD + kb * 8192u + sw128_off(t, kc)) =
                f32_to_bf16(kv * __expf(Gb - gl[u]));  // e^{G_bt - g_t} <= e^80
            const float ke3 = kv * E3[u];
            if (bt == 0) {
                *reinterpret_cast<uint16_t*>(sm + IX_KB1 + kb * 2048u + sw128_off(t, kc)) = f32_to_bf16(ke3);
                *reinterpret_cast<uint16_t*>(sm + IX_KB2 + kb * 4096u + sw128_off(t, kc)) =
                    f32_to_bf16(ke3 * f21);
                *reinterpret_cast<uint16_t*>(sm + IX_KB3 + kb * 6144u + sw128_off(t, kc)) =
                    f32_to_bf16(ke3 * f31);
            } else if (bt == 1) {
                *reinterpret_cast<uint16_t*>(sm + IX_KB2 + kb * 4096u + sw128_off(t, kc)) = f32_to_bf16(ke3);
                *reinterpret_cast<uint16_t*>(sm + IX_KB3 + kb * 6144u + sw128_off(t, kc)) =
                    f32_to_bf16(ke3 * f32);
            } else if (bt == 2) {
                *reinterpret_cast<uint16_t*>(sm + IX_KB3 + kb * 6144u + sw128_off(t, kc)) = f32_to_bf16(ke3);
            }
        }
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;

    // ---- MMA round 1: [Kr;Qr] Kd^T -> cols [0,64); [Kr;Qr] Kb(b)^T -> [64,80),[80,112),[112,160)
    if (tid == 0) {
        mma_run(tm + 0, sb + IX_KQR, 128, sb + IX_KD, 64, DK, idesc_bf16(128, 64));
        mma_run(tm + 64, sb + IX_KQR, 128, sb + IX_KB1, 16, DK, idesc_bf16(128, 16));
        mma_run(tm + 80, sb + IX_KQR, 128, sb + IX_KB2, 32, DK, idesc_bf16(128, 32));
        mma_run(tm + 112, sb + IX_KQR, 128, sb + IX_KB3, 48, DK, idesc_bf16(128, 48));
        mma_commit(bar);
    }
    uint32_t phase = 0;
    mbar_wait(bar, phase, a.status);
    phase ^= 1;
    tc_fence_after();

    // ---- extract A (rows 0..63) into fp32 smem and P (rows 64..127) into the bf16 image Ph
    {
        float* sA = reinterpret_cast<float*>(sm + IY_A);
        const int r = 32 * qd + lane;
        const bool isP = r >= 64;
        const int t = r & 63, bt = t >> 4;
        const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
        auto put = [&](int s, float val) {
            if (isP) {
                *reinterpret_cast<uint16_t*>(sm + IX_PH + sw128_off(t, s)) = f32_to_bf16(val);
            } else {
                sA[t * 64 + s] = val;
            }
        };
        if (half == 0) {
            // diagonal tile and the zero upper part: columns s >= 16 bt
            float d0[32], d1[32];
            tmem_ld32(lane_addr + 0, d0);
            tmem_ld32(lane_addr + 32, d1);
            tmem_ld_wait();
#pragma unroll
            for (int s = 0; s < 64; ++s) {
                const float val = (s < 32) ? d0[s & 31] : d1[s & 31];
                if ((s >> 4) >= bt) {
                    const bool keep = ((s >> 4) == bt) && (isP ? (s <= t) : (s < t));
                    put(s, keep ? val : 0.f);
                }
            }
        } else {
            // off-diagonal tiles: columns s < 16 bt, from the operand of this row tile
            if ((qd & 1) == 0) {  // rows t in [0, 32): tiles 0 and 1
                float d[16];
                tmem_ld16(lane_addr + 64, d);
                tmem_ld_wait();
                if (bt == 1) {
#pragma unroll
                    for (int s = 0; s < 16; ++s) put(s, d[s]);
                }
            } else {  // rows t in [32, 64): tiles 2 and 3
                float d2[32], d3[32], d3b[16];
                tmem_ld32(lane_addr + 80, d2);
                tmem_ld32(lane_addr + 112, d3);
                tmem_ld16(lane_addr + 144, d3b);
                tmem_ld_wait();
                if (bt == 2) {
#pragma unroll
                    for (int s = 0; s < 32; ++s) put(s, d2[s]);
                } else {
#pragma unroll
                    for (int s = 0; s < 48; ++s) put(s, (s < 32) ? d3[s & 31] : d3b[s & 15]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- T = (I + Diag(beta) A)^-1 Diag(beta), fp32, blocked on 16x16 tiles
    {
        float* sA = reinterpret_cast<float*>(sm + IY_A);  // becomes N = Diag(beta) A in place
        float* sX = reinterpret_cast<float*>(sm + IY_X);  // X = (I + N)^-1
        float* sY = reinterpret_cast<float*>(sm + IX_TMP);  // [3][16][16] temporaries
        for (int e = tid; e < 64 * 64; e += 256) {
            const int i = e >> 6;
            sA[e] *= s_beta[i];
        }
        __syncthreads();
        // diagonal blocks: thread per (block, column) does forward substitution
        if (tid < 64) {
            const int b = tid >> 4, j = tid & 15;
            const float* Nb = sA + (16 * b) * 64 + 16 * b;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m)
                    if (m >= j) acc += Nb[i * 64 + m] * x[m];
                x[i] = (i < j) ? 0.f : ((i == j) ? 1.f : -acc);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sX[(16 * b + i) * 64 + 16 * b + j] = x[i];
        }
        // zero the strictly upper blocks of X
        for (int e = tid; e < 64 * 64; e += 256) {
            const int i = e >> 6, j = e & 63;
            if ((j >> 4) > (i >> 4)) sX[e] = 0.f;
        }
        __syncthreads();
        // off-diagonal blocks by distance d = bi - bj:
        //   X_ij = -X_ii * sum_{m=j}^{i-1} N_im X_mj
        for (int d = 1; d <= 3; ++d) {
            const int nblk = 4 - d;
            for (int e = tid; e < nblk * 256; e += 256) {
                const int p = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int bj = p, bi = p + d;
                float acc = 0.f;
                for (int m = bj; m < bi; ++m) {
#pragma unroll
                    for (int uu = 0; uu < 16; ++uu)
                        acc += sA[(16 * bi + r) * 64 + 16 * m + uu] * sX[(16 * m + uu) * 64 + 16 * bj + cc];
                }
                sY[p * 256 + r * 16 + cc] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nblk * 256; e += 256) {
                const int p = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int bj = p, bi = p + d;
                float acc = 0.f;
#pragma unroll
                for (int uu = 0; uu < 16; ++uu)
                    acc += sX[(16 * bi + r) * 64 + 16 * bi + uu] * sY[p * 256 + uu * 16 + cc];
                sX[(16 * bi + r) * 64 + 16 * bj + cc] = -acc;
            }
            __syncthreads();
        }
        // T = X Diag(beta) -> bf16 image Ti [t][s]
        for (int e = tid; e < 64 * 64; e += 256) {
            const int t = e >> 6, s = e & 63;
            *reinterpret_cast<uint16_t*>(sm + IX_TI + sw128_off(t, s)) = f32_to_bf16(sX[e] * s_beta[s]);
        }
    }

    // ---- phase 2 operands (transposed, K = token): KGt = (K o Gam)^T, Vt = V^T, Ktt = Kt^T
    {
        // tiles of this half: bt = 2*half + lb, lb in {0, 1}
        const float eG[2] = {__expf(half ? G[2] : G[0]), __expf(half ? G[3] : G[1])};
        const float eC[2] = {__expf(G[4] - (half ? G[3] : G[1])), __expf(G[4] - (half ? G[4] : G[2]))};
        const size_t vbase = ((size_t)t0 * H + h) * DV + c;
#pragma unroll
        for (int m = 0; m < 4; ++m) {  // 8 consecutive tokens per 16-byte chunk
            uint32_t pk[4], pv[4], pt[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                float kgv[2], vvv[2], ktv[2];
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int u = 8 * m + 2 * p + e2;
                    const int t = 32 * half + u;
                    const int lb = u >> 4;  // tile within this half
                    const float kv = (t < L) ? ld_in<IN_BF16>(a.k, ebase + (size_t)t * rowstride) : 0.f;
                    const float vv = (t < L) ? ld_in<IN_BF16>(a.v, vbase + (size_t)t * H * DV) : 0.f;
                    kgv[e2] = kv * E1[u] * eG[lb];
                    ktv[e2] = kv * E3[u] * eC[lb];
                    vvv[e2] = vv;
                }
                pk[p] = pack_bf16x2(kgv[0], kgv[1]);
                pv[p] = pack_bf16x2(vvv[0], vvv[1]);
                pt[p] = pack_bf16x2(ktv[0], ktv[1]);
            }
            const uint32_t s0 = (uint32_t)(32 * half + 8 * m);
            const uint32_t off = sw128_off((uint32_t)c, s0);
            *reinterpret_cast<uint4*>(sm + IX_KGT + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(sm + IX_VT + off) = make_uint4(pv[0], pv[1], pv[2], pv[3]);
            *reinterpret_cast<uint4*>(sm + IX_KTT + off) = make_uint4(pt[0], pt[1], pt[2], pt[3]);
        }
        if (half == 1) a.ws_G[slot * DK + c] = __expf(G[4]);
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();

    // ---- MMA round 2: Wt = KGt Ti^T -> cols [0,64);  Ut = Vt Ti^T -> cols [64,128)
    if (tid == 0) {
        mma_run(tm + 0, sb + IX_KGT, 128, sb + IX_TI, 64, CH, idesc_bf16(128, 64));
        mma_run(tm + 64, sb + IX_VT, 128, sb + IX_TI, 64, CH, idesc_bf16(128, 64));
        mma_commit(bar);
    }
    mbar_wait(bar, phase, a.status);
    phase ^= 1;
    tc_fence_after();
    {
        // half 0 extracts Wt, half 1 extracts Ut; row = channel c, 64 token columns
        const uint32_t col0 = half ? 64u : 0u;
        const uint32_t dst = half ? IY_UT : IY_WT;
        float d0[32], d1[32];
        const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
        tmem_ld32(lane_addr + col0, d0);
        tmem_ld32(lane_addr + col0 + 32, d1);
        tmem_ld_wait();
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float* src = (m < 4) ? d0 : d1;
            const int o8 = (m & 3) * 8;
            const uint4 pk = make_uint4(pack_bf16x2(src[o8 + 0], src[o8 + 1]), pack_bf16x2(src[o8 + 2], src[o8 + 3]),
                                        pack_bf16x2(src[o8 + 4], src[o8 + 5]), pack_bf16x2(src[o8 + 6], src[o8 + 7]));
            *reinterpret_cast<uint4*>(sm + dst + sw128_off((uint32_t)c, (uint32_t)(8 * m))) = pk;
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA round 3: Mlr = Ktt Wt^T -> [0,128);  (P W)^T = Wt Ph^T -> [128,192);
    //                   Ob^T = Ut Ph^T -> [192,256)
    if (tid == 0) {
        mma_run(tm + 0, sb + IX_KTT, 128, sb + IY_WT, 128, CH, idesc_bf16(128, 128));
        mma_run(tm + 128, sb + IY_WT, 128, sb + IX_PH, 64, CH, idesc_bf16(128, 64));
        mma_run(tm + 192, sb + IY_UT, 128, sb + IX_PH, 64, CH, idesc_bf16(128, 64));
        mma_commit(bar);
    }
    mbar_wait(bar, phase, a.status);
    phase ^= 1;
    tc_fence_after();
    {
        const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
        // Mlr row c -> K-major SW128 image in the workspace (half h covers K block h)
        {
            uint8_t* dstM = a.ws_M + slot * SLOT_M + (size_t)half * (DK * 128);
            float d0[32], d1[32];
            tmem_ld32(lane_addr + 64 * half, d0);
            tmem_ld32(lane_addr + 64 * half + 32, d1);
            tmem_ld_wait();
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float* src = (m < 4) ? d0 : d1;
                const int o8 = (m & 3) * 8;
                const uint4 pk = make_uint4(pack_bf16x2(src[o8 + 0], src[o8 + 1]), pack_bf16x2(src[o8 + 2], src[o8 + 3]),
                                            pack_bf16x2(src[o8 + 4], src[o8 + 5]), pack_bf16x2(src[o8 + 6], src[o8 + 7]));
                *reinterpret_cast<uint4*>(dstM + sw128_off((uint32_t)c, (uint32_t)(8 * m))) = pk;
            }
        }
        // Qp^T[c][t] = scale q_tc e^{g_tc} - (P W)^T[c][t] and Ob^T[j][t]; thread covers its 32 tokens
        {
            float pw[32], ob[32];
            tmem_ld32(lane_addr + 128 + 32 * half, pw);
            tmem_ld32(lane_addr + 192 + 32 * half, ob);
            tmem_ld_wait();
            const float eG[2] = {__expf(half ? G[2] : G[0]), __expf(half ? G[3] : G[1])};
            uint8_t* dstQ = a.ws_Q + slot * SLOT_Q + (size_t)(c >> 6) * (CH * 128);
            uint16_t* dstO = reinterpret_cast<uint16_t*>(a.ws_O + slot * SLOT_O);
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int t = 32 * half + u;
                const float qv = (t < L) ? ld_in<IN_BF16>(a.q, ebase + (size_t)t * rowstride) : 0.f;
                const float qg = qv * E1[u] * eG[u >> 4] * a.scale;
                *reinterpret_cast<uint16_t*>(dstQ + sw128_off((uint32_t)t, (uint32_t)(c & 63))) =
                    f32_to_bf16(qg - pw[u]);
                dstO[(size_t)t * DV + c] = f32_to_bf16(ob[u]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA round 4: Bm = Ktt Ut^T -> cols [0,128)
    if (tid == 0) {
        mma_run(tm + 0, sb + IX_KTT, 128, sb + IY_UT, 128, CH, idesc_bf16(128, 128));
        mma_commit(bar);
    }
    mbar_wait(bar, phase, a.status);
    phase ^= 1;
    tc_fence_after();
    {
        const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
        float d0[32], d1[32];
        tmem_ld32(lane_addr + 64 * half, d0);
        tmem_ld32(lane_addr + 64 * half + 32, d1);
        tmem_ld_wait();
        uint8_t* dstB = a.ws_B + slot * SLOT_B + ((size_t)c * DV + 64 * half) * 2;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float* src = (m < 4) ? d0 : d1;
            const int o8 = (m & 3) * 8;
            const uint4 pk = make_uint4(pack_bf16x2(src[o8 + 0], src[o8 + 1]), pack_bf16x2(src[o8 + 2], src[o8 + 3]),
                                        pack_bf16x2(src[o8 + 4], src[o8 + 5]), pack_bf16x2(src[o8 + 6], src[o8 + 7]));
            *reinterpret_cast<uint4*>(dstB + 16 * m) = pk;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, INTRA_TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// chain_kernel
// ---------------------------------------------------------------------------
// Threads: 128; thread c owns state row c of the 32-column slice (32 fp32
// registers).  TMEM: 64 columns, D_S = Mlr S in [0,32) (M=128, lane = row c),
// D_O = Qp S in [32,64) (M=64: row t lives in lane 32*(t/16) + t%16).
// Shared memory: two buffers {Mlr image 32K, Qp image 16K}, the bf16 state
// operand Sb [32 value cols][128 key rows] (8K), two load barriers and one
// MMA barrier.
constexpr uint32_t CB_M = 0, CB_Q = 32768, CB_SIZE = 49152;
constexpr uint32_t C_SB = 2 * CB_SIZE;            // 98304
constexpr uint32_t C_BAR = C_SB + 8192;            // 106496
constexpr uint32_t C_TMEM = C_BAR + 24;
constexpr uint32_t CHAIN_SMEM = C_TMEM + 8 + 1024;
constexpr uint32_t CHAIN_TMEM_COLS = 64;

template <bool OUT_BF16>
__global__ void __launch_bounds__(128, 1) chain_kernel(const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, h = blockIdx.y, js = blockIdx.z;
    const int H = a.H;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + C_BAR);       // [2]
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + C_BAR + 16);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + C_TMEM);

    int64_t s_beg, s_end;
    seq_range(a, n, s_beg, s_end);
    const int nchunks = (int)((s_end - s_beg + CH - 1) / CH);
    const int c_beg = a.i0;
    const int c_end = min(a.i0 + a.wc, nchunks);
    const int nit = c_end > c_beg ? c_end - c_beg : 0;

    // state slice row c, columns [32 js, 32 js + 32)
    const size_t st_off = (((size_t)n * H + h) * DK + tid) * DV + (size_t)DVS * js;
    float S[DVS];
    {
        const float* src = a.first_pass ? a.init_state : a.state_io;
        if (src) {
#pragma unroll
            for (int j = 0; j < DVS; j += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(src + st_off + j);
                S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < DVS; ++j) S[j] = 0.f;
        }
    }

    if (nit > 0) {
        if (warp == 0) {
            tmem_alloc(s_tmem, CHAIN_TMEM_COLS);
            tmem_relinquish();
        }
        if (tid == 0) {
            mbar_init(&bar_ld[0], 1);
            mbar_init(&bar_ld[1], 1);
            mbar_init(bar_mma, 1);
            fence_mbar_init();
        }
        __syncthreads();
        tc_fence_after();
        const uint32_t tm = *s_tmem;
        auto slot_of = [&](int cidx) -> size_t { return ((size_t)n * a.wc + (cidx - a.i0)) * H + h; };
        auto issue_load = [&](int it) {
            const int b = it & 1;
            const size_t sl = slot_of(c_beg + it);
            mbar_arrive_expect_tx(&bar_ld[b], (uint32_t)(SLOT_M + SLOT_Q));
            bulk_g2s(sm + b * CB_SIZE + CB_M, a.ws_M + sl * SLOT_M, (uint32_t)SLOT_M, &bar_ld[b]);
            bulk_g2s(sm + b * CB_SIZE + CB_Q, a.ws_Q + sl * SLOT_Q, (uint32_t)SLOT_Q, &bar_ld[b]);
        };
        if (tid == 0) issue_load(0);

        bool ok = true;
        int it = 0;
        for (; it < nit && ok; ++it) {
            const int cidx = c_beg + it;
            const size_t sl = slot_of(cidx);
            const int64_t t0 = s_beg + (int64_t)cidx * CH;
            const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
            if (tid == 0 && it + 1 < nit) issue_load(it + 1);

            // per-chunk inputs of this thread: Bm row slice, Gam_C, Ob row slice
            float bm[DVS];
            {
                const uint4* src = reinterpret_cast<const uint4*>(a.ws_B + sl * SLOT_B + ((size_t)tid * DV + DVS * js) * 2);
#pragma unroll
                for (int m = 0; m < DVS / 8; ++m) {
                    const uint4 w = __ldg(src + m);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        bm[8 * m + 2 * p] = __uint_as_float(ww[p] << 16);
                        bm[8 * m + 2 * p + 1] = __uint_as_float(ww[p] & 0xFFFF0000u);
                    }
                }
            }
            const float gamC = __ldg(a.ws_G + sl * DK + tid);
            const int trow = 16 * warp + (lane & 15);  // output row served by this lane (lane < 16)
            float obv[DVS];
            if (lane < 16) {
                const uint4* src = reinterpret_cast<const uint4*>(a.ws_O + sl * SLOT_O + ((size_t)trow * DV + DVS * js) * 2);
#pragma unroll
                for (int m = 0; m < DVS / 8; ++m) {
                    const uint4 w = __ldg(src + m);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        obv[8 * m + 2 * p] = __uint_as_float(ww[p] << 16);
                        obv[8 * m + 2 * p + 1] = __uint_as_float(ww[p] & 0xFFFF0000u);
                    }
                }
            }

            // state operand Sb[j][c] = bf16(S[c][j]) (K-major: row = value col j, K = key row c)
            {
                const uint32_t kb = (uint32_t)tid >> 6, kc = (uint32_t)tid & 63u;
#pragma unroll
                for (int j = 0; j < DVS; ++j)
                    *reinterpret_cast<uint16_t*>(sm + C_SB + kb * (DVS * 128) + sw128_off((uint32_t)j, kc)) =
                        f32_to_bf16(S[j]);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == 0) {
                const int b = it & 1;
                if (mbar_wait(&bar_ld[b], (uint32_t)((it >> 1) & 1), a.status)) {
                    tc_fence_after();
                    mma_run(tm + 0, sbase + b * CB_SIZE + CB_M, 128, sbase + C_SB, DVS, DK, idesc_bf16(128, DVS));
                    mma_run(tm + 32, sbase + b * CB_SIZE + CB_Q, 64, sbase + C_SB, DVS, DK, idesc_bf16(64, DVS));
                }
                mma_commit(bar_mma);
            }
            ok = mbar_wait(bar_mma, (uint32_t)(it & 1), a.status);
            tc_fence_after();
            if (!ok) {
                // a wait gave up: let the prefetch in flight land before leaving
                if (tid == 0 && it + 1 < nit) mbar_wait(&bar_ld[(it + 1) & 1], (uint32_t)(((it + 1) >> 1) & 1), nullptr);
                break;
            }

            const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
            float ds[DVS], dO[DVS];
            tmem_ld32(lane_addr + 0, ds);
            tmem_ld32(lane_addr + 32, dO);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < DVS; ++j) S[j] = gamC * S[j] - ds[j] + bm[j];
            if (lane < 16 && trow < L) {
                const size_t obase = ((size_t)(t0 + trow) * H + h) * DV + (size_t)DVS * js;
                if constexpr (OUT_BF16) {
                    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.o) + obase);
#pragma unroll
                    for (int m = 0; m < DVS / 8; ++m) {
                        const int j = 8 * m;
                        dst[m] = make_uint4(pack_bf16x2(dO[j] + obv[j], dO[j + 1] + obv[j + 1]),
                                            pack_bf16x2(dO[j + 2] + obv[j + 2], dO[j + 3] + obv[j + 3]),
                                            pack_bf16x2(dO[j + 4] + obv[j + 4], dO[j + 5] + obv[j + 5]),
                                            pack_bf16x2(dO[j + 6] + obv[j + 6], dO[j + 7] + obv[j + 7]));
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + obase);
#pragma unroll
                    for (int m = 0; m < DVS / 4; ++m) {
                        const int j = 4 * m;
                        dst[m] = make_float4(dO[j] + obv[j], dO[j + 1] + obv[j + 1], dO[j + 2] + obv[j + 2],
                                             dO[j + 3] + obv[j + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
        }
        tc_fence_after();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tm, CHAIN_TMEM_COLS);
    }

    // write the carried / final state slice
#pragma unroll
    for (int j = 0; j < DVS; j += 4)
        *reinterpret_cast<float4*>(a.state_io + st_off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
}

// Flags cu_seqlens that contradict T, n_seqs or max_seqlen (one thread).
__global__ void check_cu_kernel(const int32_t* cu, int n_seqs, int64_t T, int64_t max_seqlen, uint32_t* status) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    bool bad = cu[0] != 0 || (int64_t)cu[n_seqs] != T;
    for (int i = 0; i < n_seqs && !bad; ++i) {
        const int64_t len = (int64_t)cu[i + 1] - (int64_t)cu[i];
        if (len < 0 || len > max_seqlen) bad = true;
    }
    if (bad) atomicOr(status, DEV_ERR_SEQLEN);
}

// ------------------------------------------------------------- host side --

size_t chunk_slot_bytes() { return SLOT_M + SLOT_Q + SLOT_B + SLOT_O + SLOT_G; }

// Fixed part of the workspace: status word (256 B) + state carry when the
// caller does not ask for the final state.
size_t chunk_fixed_bytes(int n_seqs, int H, bool need_carry) {
    size_t b = 256;
    if (need_carry) b += (size_t)n_seqs * H * DK * DV * sizeof(float);
    return b;
}

static bool g_attr_set = false;

cudaError_t chunk_fwd_launch(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, void* o, float* final_state, int B, int64_t T, int H,
                             const int32_t* cu, int n_seqs, int64_t max_seqlen, bool in_bf16, bool out_bf16,
                             float scale, void* workspace, size_t ws_bytes, cudaStream_t stream, int* n_passes) {
    cudaError_t err;
    if (!g_attr_set) {
        err = cudaFuncSetAttribute(intra_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, INTRA_SMEM);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(intra_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, INTRA_SMEM);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(chain_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, CHAIN_SMEM);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(chain_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, CHAIN_SMEM);
        if (err != cudaSuccess) return err;
        g_attr_set = true;
    }
    const int N = cu ? n_seqs : B;
    const int64_t seqT = cu ? T : T;  // tokens per sequence (fixed) / total (varlen)
    const int64_t maxlen = cu ? max_seqlen : T;
    const int nchunks_max = (int)((maxlen + CH - 1) / CH);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    const bool need_carry = final_state == nullptr;
    const size_t fixed = chunk_fixed_bytes(N, H, need_carry);
    float* carry = need_carry ? reinterpret_cast<float*>(ws + 256) : final_state;
    const size_t per_wc = (size_t)N * H * chunk_slot_bytes();
    const size_t head = (fixed + 1023) & ~(size_t)1023;
    const size_t wc_fit = ws_bytes > head ? (ws_bytes - head) / per_wc : 0;
    int wc = (int)(wc_fit < (size_t)nchunks_max ? wc_fit : (size_t)nchunks_max);
    if (wc < 1) wc = 1;
    const size_t slots = (size_t)N * wc * H;
    uint8_t* p = ws + head;
    ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.init_state = init_state; a.state_io = carry; a.o = o; a.cu = cu;
    a.ws_M = p; p += slots * SLOT_M;
    a.ws_Q = p; p += slots * SLOT_Q;
    a.ws_B = p; p += slots * SLOT_B;
    a.ws_O = p; p += slots * SLOT_O;
    a.ws_G = reinterpret_cast<float*>(p);
    a.status = status;
    a.T = cu ? T : seqT;
    a.H = H; a.n_seqs = N; a.wc = wc; a.scale = scale;

    err = cudaMemsetAsync(status, 0, 4, stream);
    if (err != cudaSuccess) return err;
    if (cu) {
        prof_begin(PROF_CHECK, stream);
        check_cu_kernel<<<1, 32, 0, stream>>>(cu, n_seqs, T, max_seqlen, status);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        prof_end(PROF_CHECK, stream);
    }
    int passes = 0;
    const int npass = nchunks_max > 0 ? (nchunks_max + wc - 1) / wc : 1;
    for (int ps = 0; ps < npass; ++ps) {
        a.i0 = ps * wc;
        a.first_pass = ps == 0;
        if (nchunks_max > 0) {
            const dim3 gi((unsigned)(N * wc), (unsigned)H);
            prof_begin(PROF_INTRA, stream);
            if (in_bf16) intra_kernel<true><<<gi, 256, INTRA_SMEM, stream>>>(a);
            else intra_kernel<false><<<gi, 256, INTRA_SMEM, stream>>>(a);
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
            prof_end(PROF_INTRA, stream);
        }
        const dim3 gc((unsigned)N, (unsigned)H, (unsigned)(DV / DVS));
        prof_begin(PROF_CHAIN, stream);
        if (out_bf16) chain_kernel<true><<<gc, 128, CHAIN_SMEM, stream>>>(a);
        else chain_kernel<false><<<gc, 128, CHAIN_SMEM, stream>>>(a);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        prof_end(PROF_CHAIN, stream);
        ++passes;
    }
    if (n_passes) *n_passes = passes;
    return cudaSuccess;
}

}  // namespace kda
