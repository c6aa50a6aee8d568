// kda_bwd.cu -- backward pass of the chunkwise KDA prefill.
//
// The pages describe no backward pass.  This is the exact gradient of the
// forward (the recurrence and its chunkwise form: K3 article summaries,
// xhh.club tag page, items "KDA recurrence form" and "chunkwise parallel
// algorithm"), arranged chunkwise:
//   1. the forward walk is recomputed without outputs; it leaves every chunk's
//      slot (M_lr, Q', Gamma_C) in the workspace and the state at every chunk
//      boundary in a checkpoint buffer;
//   2. chain_bwd_kernel walks the chunks of a sequence in reverse with
//      dS = dL/d(state at the end of chunk c):
//          dS_end[c] = dS,    dS <- Diag(Gamma_C) dS - M_lr^T dS + Q'^T dO_c
//      starting from dL/dS_final and ending with dL/dS_0;
//   3. bwd_intra_kernel takes one (chunk, head) at a time, with the chunk-start
//      state S0 and dS_C = dS_end[c], and forms dq, dk, dv, dbeta, dlog_alpha of
//      the chunk's tokens.
// Per chunk (L <= 64 tokens; g = in-chunk cumulative sum of the clamped
// log-decays, Gam = e^g, g_C = g of the last token, qb = scale q,
// K^C = K o e^{g_C - g}):
//   A_ts = sum_i k_ti k_si e^{g_ti - g_si}  (s < t),   P_ts = sum_i qb_ti k_si e^{g_ti - g_si}  (s <= t)
//   M = I + Diag(beta) A,   R = V - (K o Gam) S0,   U = M^-1 Diag(beta) R
//   dU = P^T dO + K^C dS_C,   Y = M^-T dU,   dv = Diag(beta) Y
//   dM = -(Y U^T) on s < t,   dA = Diag(beta) dM,   dbeta = rowsum(Y o R) + rowsum(dM o A)
//   dP = dO U^T on s <= t
//   the S0 terms dO S0^T (-> qb, g), -dv S0^T (-> k, g), the K^C term U dS_C^T
//   (-> k, g, g_C), Gam_C o rowsum(S0 o dS_C) (-> g_C), and the A / P
//   contractions (-> q, k, g); dlog_alpha = reverse cumulative sum of dg over the
//   chunk, zero where log_alpha < -5 (the clamp passes the gradient where
//   log_alpha >= -5).
// The A / P terms use per-16-token-block reference points r (the block's first
// token): e^{g_t - g_s} = e^{g_t - g_r} e^{g_r - g_s}, so each exponential is
// formed once per (token, channel, block) and never overflows.
// Everything is fp32 on the CUDA cores.
#include "kda_launch.h"
#include "kda_profile.h"
#include "kda_slots.h"
#include "kda_sm100.cuh"

namespace kda {

struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* log_alpha;
    const void* beta;
    const void* d_o;
    const float* init_state;   // nullable
    const float* d_final;      // nullable
    float* d_init;             // nullable
    float* dq;
    float* dk;
    float* dv;
    float* dla;
    float* dbeta;
    const int32_t* cu;         // nullable (fixed length)
    const uint8_t* slots;      // forward chunk slots [n_seqs][wc][H]
    const float* ckpt;         // states after every whole chunk [n_seqs][n_ckpt][H][dk][dv]
    float* ds_end;             // dL/d(state at chunk end) [n_seqs][wc][H][dk][dv]
    uint32_t* status;
    int64_t T;
    int H, n_seqs, wc, n_ckpt;
    float scale;
    int in_bf16;
};

namespace {

constexpr int STATE = DK * DV;  // elements of one state

KDA_DEV void bwd_seq_range(const BwdArgs& a, int n, int64_t& sb, int64_t& se) {
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

KDA_DEV float ld_in(const void* p, size_t idx, int bf16) {
    if (bf16) return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p) + idx) << 16);
    return __ldg(reinterpret_cast<const float*>(p) + idx);
}

// ------------------------------------------------------------ reverse chain
constexpr int CB_THREADS = 512;  // thread = (key row i = tid % 128, 8-column group tid / 128)
constexpr uint32_t CB_SLOT = SO_MQG;                 // M_lr + Q' + Gamma_C of one chunk
constexpr uint32_t CB_DS = 2 * CB_SLOT;              // dS [128][32] fp32
constexpr uint32_t CB_DO = CB_DS + DK * DVS * 4;     // dO [64][32] fp32
constexpr uint32_t CB_BAR = CB_DO + CH * DVS * 4;    // two mbarriers
constexpr uint32_t CB_SMEM = CB_BAR + 16 + 128;

__global__ void __launch_bounds__(CB_THREADS, 1) chain_bwd_kernel(const BwdArgs a) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int js = blockIdx.x, h = blockIdx.y, n = blockIdx.z, H = a.H;
    const int tid = threadIdx.x, i = tid & (DK - 1), cq = tid >> 7;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + CB_BAR);
    float* sdS = reinterpret_cast<float*>(sm + CB_DS);
    float* sdO = reinterpret_cast<float*>(sm + CB_DO);
    int64_t s_beg, s_end;
    bwd_seq_range(a, n, s_beg, s_end);
    const int nck = (int)((s_end - s_beg + CH - 1) / CH);
    const size_t st = ((size_t)n * H + h) * STATE + (size_t)i * DV + DVS * js + 8 * cq;  // this thread's 8 values
    float dS[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) dS[j] = a.d_final ? a.d_final[st + j] : 0.f;
    auto slot = [&](int c) { return a.slots + (((size_t)n * a.wc + c) * H + h) * SLOT_BYTES; };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        for (int r = 0; r < 2 && r < nck; ++r) {
            mbar_arrive_expect_tx(&bar[r], CB_SLOT);
            bulk_g2s(sm + r * CB_SLOT, slot(nck - 1 - r), CB_SLOT, &bar[r]);
        }
    }
    __syncthreads();
    int issued = nck < 2 ? nck : 2, waited = 0;
    bool failed = false;
    // this thread's 4 values of a chunk's dO slice: token tid / 8, columns 4 (tid % 8) ..
    auto load_dO = [&](int c) {
        const int t = tid >> 3, c4 = (tid & 7) * 4;
        const int64_t tc = s_beg + (int64_t)c * CH + t;
        if (c < 0 || tc >= s_end) return make_float4(0.f, 0.f, 0.f, 0.f);
        const size_t base = ((size_t)tc * H + h) * DV + DVS * js + c4;
        return make_float4(ld_in(a.d_o, base, a.in_bf16), ld_in(a.d_o, base + 1, a.in_bf16),
                           ld_in(a.d_o, base + 2, a.in_bf16), ld_in(a.d_o, base + 3, a.in_bf16));
    };
    float4 dO_next = load_dO(nck - 1);
    uint32_t m_off[8];  // sw128_off(mm, i & 63) for mm = 0..7
#pragma unroll
    for (int mm = 0; mm < 8; ++mm) m_off[mm] = sw128_off((uint32_t)mm, (uint32_t)(i & 63));
    for (int r = 0; r < nck; ++r) {
        const int c = nck - 1 - r, b = r & 1;
        const int64_t t0 = s_beg + (int64_t)c * CH;
        const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
        // dS at the end of chunk c
        float* dst = a.ds_end + (((size_t)n * a.wc + c) * H + h) * STATE + (size_t)i * DV + DVS * js + 8 * cq;
        reinterpret_cast<float4*>(dst)[0] = make_float4(dS[0], dS[1], dS[2], dS[3]);
        reinterpret_cast<float4*>(dst)[1] = make_float4(dS[4], dS[5], dS[6], dS[7]);
        reinterpret_cast<float4*>(sdS + i * DVS + 8 * cq)[0] = make_float4(dS[0], dS[1], dS[2], dS[3]);
        reinterpret_cast<float4*>(sdS + i * DVS + 8 * cq)[1] = make_float4(dS[4], dS[5], dS[6], dS[7]);
        // dO slice of chunk c ([64 tokens][32 columns]), loaded during the previous iteration
        *reinterpret_cast<float4*>(sdO + (tid >> 3) * DVS + (tid & 7) * 4) = dO_next;
        const bool ok = mbar_wait(&bar[b], (uint32_t)((r >> 1) & 1), a.status);
        if (!__syncthreads_and(ok)) {
            failed = true;
            break;
        }
        waited = r + 1;
        const uint8_t* buf = sm + b * CB_SLOT;
        const float gam = *reinterpret_cast<const float*>(buf + SO_G + 4 * i);
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = gam * dS[j];
        // - M_lr^T dS: column i of M_lr against every row of dS.  Element (m, i) of the
        // K-major SW128 image sits at (i >> 6) * 16384 + sw128_off(m, i & 63); for
        // m = 8 m8 + mm that is m8 * 1024 + off[mm], with off[] fixed per thread.
        const uint8_t* mcol = buf + SO_M + (size_t)(i >> 6) * 16384;
        for (int m8 = 0; m8 < DK / 8; ++m8) {
            const uint8_t* mrow = mcol + m8 * 1024;
            const float* drow = sdS + m8 * 8 * DVS + 8 * cq;
#pragma unroll
            for (int mm = 0; mm < 8; ++mm) {
                const uint16_t bits = *reinterpret_cast<const uint16_t*>(mrow + m_off[mm]);
                const float mv = __uint_as_float((uint32_t)bits << 16);
                const float4 d0 = reinterpret_cast<const float4*>(drow + mm * DVS)[0];
                const float4 d1 = reinterpret_cast<const float4*>(drow + mm * DVS)[1];
                acc[0] -= mv * d0.x; acc[1] -= mv * d0.y; acc[2] -= mv * d0.z; acc[3] -= mv * d0.w;
                acc[4] -= mv * d1.x; acc[5] -= mv * d1.y; acc[6] -= mv * d1.z; acc[7] -= mv * d1.w;
            }
        }
        // + Q'^T dO: column i of Q' against every token row of dO
        const uint8_t* qcol = buf + SO_Q + (size_t)(i >> 3) * 1024 + (i & 7) * 16;
        for (int t = 0; t < L; ++t) {
            const uint16_t bits = *reinterpret_cast<const uint16_t*>(qcol + (t >> 3) * 128 + (t & 7) * 2);
            const float qv = __uint_as_float((uint32_t)bits << 16);
            const float4 o0 = reinterpret_cast<const float4*>(sdO + t * DVS + 8 * cq)[0];
            const float4 o1 = reinterpret_cast<const float4*>(sdO + t * DVS + 8 * cq)[1];
            acc[0] += qv * o0.x; acc[1] += qv * o0.y; acc[2] += qv * o0.z; acc[3] += qv * o0.w;
            acc[4] += qv * o1.x; acc[5] += qv * o1.y; acc[6] += qv * o1.z; acc[7] += qv * o1.w;
        }
        dO_next = load_dO(c - 1);
        __syncthreads();  // buffer b, dS and dO are no longer read
        if (tid == 0 && r + 2 < nck) {
            mbar_arrive_expect_tx(&bar[b], CB_SLOT);
            bulk_g2s(sm + b * CB_SLOT, slot(nck - 1 - (r + 2)), CB_SLOT, &bar[b]);
            issued = r + 3;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) dS[j] = acc[j];
    }
    if (failed && tid == 0) {
        // copies still in flight land before the CTA retires (bounded)
        for (int r = waited; r < issued; ++r) mbar_wait(&bar[r & 1], (uint32_t)((r >> 1) & 1), nullptr);
    }
    if (!failed && a.d_init) {
        float* dst = a.d_init + st;
        reinterpret_cast<float4*>(dst)[0] = make_float4(dS[0], dS[1], dS[2], dS[3]);
        reinterpret_cast<float4*>(dst)[1] = make_float4(dS[4], dS[5], dS[6], dS[7]);
    }
}

// -------------------------------------------------------- chunk-local part
constexpr int BI_THREADS = 512;
constexpr int LP = 65;    // padded row of the 64 x 64 matrices
constexpr int FP = 132;   // padded row of the factor buffer
constexpr int QP = 33;    // padded row of the 64 x 32 quarter buffers
constexpr int NQ = 32;    // value columns per quarter
constexpr uint32_t BI_G = 0;                                  // g [64][128]
constexpr uint32_t BI_A = BI_G + CH * DK * 4;                  // A [64][65]
constexpr uint32_t BI_P = BI_A + CH * LP * 4;                  // P
constexpr uint32_t BI_MI = BI_P + CH * LP * 4;                 // M^-1
constexpr uint32_t BI_DP = BI_MI + CH * LP * 4;                // dP (accumulated)
constexpr uint32_t BI_DM = BI_DP + CH * LP * 4;                // dM (accumulated), then dA
constexpr uint32_t BI_F = BI_DM + CH * LP * 4;                 // factors [128][132]
constexpr uint32_t BI_R = BI_F + 128 * FP * 4;                 // R quarter [64][33]
constexpr uint32_t BI_U = BI_R + CH * QP * 4;                  // U quarter
constexpr uint32_t BI_DU = BI_U + CH * QP * 4;                 // dU quarter, then Y
constexpr uint32_t BI_DO = BI_DU + CH * QP * 4;                // dO quarter
constexpr uint32_t BI_BETA = BI_DO + CH * QP * 4;              // beta [64]
constexpr uint32_t BI_DB = BI_BETA + 256;                      // rowsum(Y o R) [64]
constexpr uint32_t BI_GC = BI_DB + 256;                        // g_C [128]
constexpr uint32_t BI_DGC = BI_GC + 512;                       // dL/dg_C [128]
constexpr uint32_t BI_SMEM = BI_DGC + 512;

// Factor rows of block bt (reference token r = 16 bt) in the factor buffer:
// rows [0, 16 bt + 16): Kout_s = k_s o e^{g_r - g_s};  rows [64, 80): Kin_t = k_t o
// e^{g_t - g_r};  rows [80, 96): Qin_t = qb_t o e^{g_t - g_r}  (t in the block).
KDA_DEV void build_factors(const BwdArgs& a, float* sF, const float* sG, int bt, int64_t t0, int L, int h,
                           int tid) {
    const int r = 16 * bt, ns = 16 * bt + 16;
    const int n_el = (ns + 32) * DK;  // a multiple of 4 * BI_THREADS
    for (int e0 = tid; e0 < n_el; e0 += 4 * BI_THREADS) {
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // loads first, all four in flight
            const int e = e0 + u * BI_THREADS, row = e >> 7, i = e & (DK - 1);
            const int t = row < ns ? row : r + ((row - ns) & 15);
            x[u] = 0.f;
            if (t < L) {
                const size_t idx = ((size_t)(t0 + t) * a.H + h) * DK + i;
                x[u] = (row < ns + 16) ? ld_in(a.k, idx, a.in_bf16) : a.scale * ld_in(a.q, idx, a.in_bf16);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * BI_THREADS, row = e >> 7, i = e & (DK - 1);
            const float gr = sG[r * DK + i];
            if (row < ns) {
                sF[row * FP + i] = x[u] * __expf(gr - sG[row * DK + i]);
            } else {
                const int tt = row - ns;  // 0..31: Kin rows, then Qin rows
                const int t = r + (tt & 15);
                sF[(64 + tt) * FP + i] = x[u] * __expf(sG[t * DK + i] - gr);
            }
        }
    }
}

// Pulls an item's token rows (q, k, v, log_alpha, dO: 64 rows each), its
// chunk-start state and its end-of-chunk state gradient into L2 ahead of use.
KDA_DEV void prefetch_item(const BwdArgs& a, int64_t item, int64_t n_items, int tid) {
    if (item >= n_items) return;
    const int H = a.H;
    const int h = (int)(item % H);
    const int c = (int)((item / H) % a.wc);
    const int n = (int)(item / ((int64_t)H * a.wc));
    int64_t s_beg, s_end;
    bwd_seq_range(a, n, s_beg, s_end);
    const int64_t t0 = s_beg + (int64_t)c * CH;
    if (t0 >= s_end) return;
    const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
    const size_t esz = a.in_bf16 ? 2 : 4, row = DK * esz;  // bytes of one head row
    const int lines_row = (int)(row / 128);
    const void* tens[5] = {a.q, a.k, a.v, a.log_alpha, a.d_o};
    for (int e = tid; e < 5 * CH * lines_row; e += BI_THREADS) {
        const int tsr = e / (CH * lines_row), rem = e % (CH * lines_row), t = rem / lines_row, ln = rem % lines_row;
        if (t >= L) continue;
        const char* p = reinterpret_cast<const char*>(tens[tsr]) + ((size_t)(t0 + t) * H + h) * row + ln * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
    }
    const float* S0 = c == 0 ? (a.init_state ? a.init_state + ((size_t)n * H + h) * STATE : nullptr)
                             : a.ckpt + (((size_t)n * a.n_ckpt + (c - 1)) * H + h) * STATE;
    const float* dSC = a.ds_end + (((size_t)n * a.wc + c) * H + h) * STATE;
    for (int e = tid; e < 2 * STATE * 4 / 128; e += BI_THREADS) {
        const int which = e / (STATE * 4 / 128), ln = e % (STATE * 4 / 128);
        const float* base = which ? dSC : S0;
        if (base) asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(base) + (size_t)ln * 128));
    }
}

__global__ void __launch_bounds__(BI_THREADS, 1) bwd_intra_kernel(const BwdArgs a, int64_t n_items) {
    extern __shared__ __align__(128) uint8_t sm[];
    float* sG = reinterpret_cast<float*>(sm + BI_G);
    float* sA = reinterpret_cast<float*>(sm + BI_A);
    float* sP = reinterpret_cast<float*>(sm + BI_P);
    float* sMi = reinterpret_cast<float*>(sm + BI_MI);
    float* sdP = reinterpret_cast<float*>(sm + BI_DP);
    float* sdM = reinterpret_cast<float*>(sm + BI_DM);
    float* sF = reinterpret_cast<float*>(sm + BI_F);
    float* sR = reinterpret_cast<float*>(sm + BI_R);
    float* sU = reinterpret_cast<float*>(sm + BI_U);
    float* sDU = reinterpret_cast<float*>(sm + BI_DU);
    float* sDO = reinterpret_cast<float*>(sm + BI_DO);
    float* sBeta = reinterpret_cast<float*>(sm + BI_BETA);
    float* sDb = reinterpret_cast<float*>(sm + BI_DB);
    float* sGC = reinterpret_cast<float*>(sm + BI_GC);
    float* sDgC = reinterpret_cast<float*>(sm + BI_DGC);
    const int tid = threadIdx.x, H = a.H;
    // register-owned elements: tokens 4 tg .. 4 tg + 3, key channels ig + 32 y (y = 0..3;
    // interleaved so that a warp's 32 lanes touch 32 consecutive channels)
    const int tg = tid >> 5, ig = tid & 31;

    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int h = (int)(item % H);
        const int c = (int)((item / H) % a.wc);
        const int n = (int)(item / ((int64_t)H * a.wc));
        int64_t s_beg, s_end;
        bwd_seq_range(a, n, s_beg, s_end);
        const int64_t t0 = s_beg + (int64_t)c * CH;
        if (t0 >= s_end) continue;  // uniform over the CTA
        const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
        const int nb = (L + 15) >> 4;
        const float* S0 = c == 0 ? (a.init_state ? a.init_state + ((size_t)n * H + h) * STATE : nullptr)
                                 : a.ckpt + (((size_t)n * a.n_ckpt + (c - 1)) * H + h) * STATE;
        const float* dSC = a.ds_end + (((size_t)n * a.wc + c) * H + h) * STATE;
        prefetch_item(a, item + gridDim.x, n_items, tid);  // the next item's inputs into L2

        // ---- P0: beta, g (cumulative clamped log-decay), zeroed accumulators
        if (tid < CH) {
            sBeta[tid] = tid < L ? ld_in(a.beta, (size_t)(t0 + tid) * H + h, a.in_bf16) : 0.f;
            sDb[tid] = 0.f;
        }
        if (tid < DK) {
            float lv[CH];  // all loads in flight at once
#pragma unroll
            for (int t = 0; t < CH; ++t)
                lv[t] = t < L ? fmaxf(ld_in(a.log_alpha, ((size_t)(t0 + t) * H + h) * DK + tid, a.in_bf16), -5.f) : 0.f;
            float g = 0.f;
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                g += lv[t];
                sG[t * DK + tid] = g;
            }
            sGC[tid] = g;
            sDgC[tid] = 0.f;
        }
        for (int e = tid; e < CH * LP; e += BI_THREADS) {
            sA[e] = 0.f; sP[e] = 0.f; sdP[e] = 0.f; sdM[e] = 0.f;
        }
        __syncthreads();

        // ---- P1: A (s < t) and P (s <= t), block row by block row
        for (int bt = 0; bt < nb; ++bt) {
            build_factors(a, sF, sG, bt, t0, L, h, tid);
            __syncthreads();
            const int ns = 16 * bt + 16;
            for (int e = tid; e < 16 * ns; e += BI_THREADS) {
                const int tl = e & 15, s = e >> 4, t = 16 * bt + tl;
                if (t >= L || s > t) continue;
                const float* kin = sF + (64 + tl) * FP;
                const float* qin = sF + (80 + tl) * FP;
                const float* ko = sF + s * FP;
                float da = 0.f, dp = 0.f;
#pragma unroll 8
                for (int i4 = 0; i4 < DK; i4 += 4) {
                    const float4 kv = *reinterpret_cast<const float4*>(ko + i4);
                    const float4 x = *reinterpret_cast<const float4*>(kin + i4);
                    const float4 y = *reinterpret_cast<const float4*>(qin + i4);
                    da += x.x * kv.x + x.y * kv.y + x.z * kv.z + x.w * kv.w;
                    dp += y.x * kv.x + y.y * kv.y + y.z * kv.z + y.w * kv.w;
                }
                if (s < t) sA[t * LP + s] = da;
                sP[t * LP + s] = dp;
            }
            __syncthreads();
        }

        // ---- P2: M^-1, M = I + Diag(beta) A (unit lower triangular): column cc by the
        // 8 lanes tid / 8 == cc, forward substitution down the rows, the sum over earlier
        // rows split over the lanes and reduced by shuffles (all lanes take part in every
        // shuffle; loop trip counts differ, the warp reconverges before them)
        {
            const int cc = tid >> 3, part = tid & 7;
            for (int t = 0; t < CH; ++t) {
                float p = 0.f;
                for (int s = cc + part; s < t; s += 8) p += sA[t * LP + s] * sMi[s * LP + cc];
                p += __shfl_xor_sync(0xFFFFFFFFu, p, 1);
                p += __shfl_xor_sync(0xFFFFFFFFu, p, 2);
                p += __shfl_xor_sync(0xFFFFFFFFu, p, 4);
                const float x = t < cc ? 0.f : (t == cc ? 1.f : -sBeta[t] * p);
                if (part == 0) sMi[t * LP + cc] = x;
                __syncwarp();
            }
        }
        // factors K o Gam (rows 0-63) and K^C = K o e^{g_C - g} (rows 64-127)
        for (int e0 = tid; e0 < CH * DK; e0 += 4 * BI_THREADS) {
            float kv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * BI_THREADS, t = e >> 7, i = e & (DK - 1);
                kv[u] = t < L ? ld_in(a.k, ((size_t)(t0 + t) * H + h) * DK + i, a.in_bf16) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * BI_THREADS, t = e >> 7, i = e & (DK - 1);
                const float g = sG[t * DK + i];
                sF[t * FP + i] = kv[u] * __expf(g);
                sF[(64 + t) * FP + i] = kv[u] * __expf(sGC[i] - g);
            }
        }
        __syncthreads();

        float aQG[4][4], aKG[4][4], aKC[4][4], rowS[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            rowS[x] = 0.f;
#pragma unroll
            for (int y = 0; y < 4; ++y) aQG[x][y] = aKG[x][y] = aKC[x][y] = 0.f;
        }

        // ---- P3: value columns in quarters of 32
        for (int qd = 0; qd < DV / NQ; ++qd) {
            const int j0 = NQ * qd;
            // (a) dO quarter and R = V - (K o Gam) S0
            {
                const int t = tid >> 3, jq = (tid & 7) * 4;
                float r4[4] = {0.f, 0.f, 0.f, 0.f}, o4[4] = {0.f, 0.f, 0.f, 0.f};
                if (t < L) {
                    const size_t base = ((size_t)(t0 + t) * H + h) * DV + j0 + jq;
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        r4[x] = ld_in(a.v, base + x, a.in_bf16);
                        o4[x] = ld_in(a.d_o, base + x, a.in_bf16);
                    }
                    if (S0) {
                        const float* kg = sF + t * FP;
#pragma unroll 8
                        for (int i = 0; i < DK; ++i) {
                            const float4 s4 = __ldg(reinterpret_cast<const float4*>(S0 + (size_t)i * DV + j0 + jq));
                            const float w = kg[i];
                            r4[0] -= w * s4.x; r4[1] -= w * s4.y; r4[2] -= w * s4.z; r4[3] -= w * s4.w;
                        }
                    }
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    sR[t * QP + jq + x] = r4[x];
                    sDO[t * QP + jq + x] = o4[x];
                }
            }
            __syncthreads();
            // (b) U = M^-1 Diag(beta) R;  dU = P^T dO + K^C dS_C
            {
                const int t = tid >> 3, jq = (tid & 7) * 4;
                float u4[4] = {0.f, 0.f, 0.f, 0.f}, d4[4] = {0.f, 0.f, 0.f, 0.f};
                for (int s = 0; s <= t; ++s) {
                    const float w = sMi[t * LP + s] * sBeta[s];
#pragma unroll
                    for (int x = 0; x < 4; ++x) u4[x] += w * sR[s * QP + jq + x];
                }
                for (int tt = t; tt < CH; ++tt) {
                    const float w = sP[tt * LP + t];
#pragma unroll
                    for (int x = 0; x < 4; ++x) d4[x] += w * sDO[tt * QP + jq + x];
                }
                const float* kc = sF + (64 + t) * FP;
#pragma unroll 8
                for (int i = 0; i < DK; ++i) {
                    const float4 s4 = __ldg(reinterpret_cast<const float4*>(dSC + (size_t)i * DV + j0 + jq));
                    const float w = kc[i];
                    d4[0] += w * s4.x; d4[1] += w * s4.y; d4[2] += w * s4.z; d4[3] += w * s4.w;
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    sU[t * QP + jq + x] = u4[x];
                    sDU[t * QP + jq + x] = d4[x];
                }
            }
            __syncthreads();
            // (c) Y = M^-T dU; dv = beta Y; rowsum(Y o R)
            {
                const int t = tid >> 3, jq = (tid & 7) * 4;
                float y4[4] = {0.f, 0.f, 0.f, 0.f};
                for (int s = t; s < CH; ++s) {
                    const float w = sMi[s * LP + t];
#pragma unroll
                    for (int x = 0; x < 4; ++x) y4[x] += w * sDU[s * QP + jq + x];
                }
                float yr = 0.f;
#pragma unroll
                for (int x = 0; x < 4; ++x) yr += y4[x] * sR[t * QP + jq + x];
                atomicAdd(&sDb[t], yr);
                if (t < L) {
                    const float b = sBeta[t];
                    float4* dst = reinterpret_cast<float4*>(a.dv + ((size_t)(t0 + t) * H + h) * DV + j0 + jq);
                    *dst = make_float4(b * y4[0], b * y4[1], b * y4[2], b * y4[3]);
                }
                __syncthreads();  // every read of dU is done
#pragma unroll
                for (int x = 0; x < 4; ++x) sDU[t * QP + jq + x] = y4[x];  // sDU now holds Y
            }
            __syncthreads();
            // (d) dP += dO U^T (s <= t);  dM -= Y U^T (s < t)
            {
                // rows s = sl + 8 x: the 8 lanes sharing t read 8 consecutive rows of U
                const int t = tid >> 3, sl = tid & 7;
                float dp[8], dm[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) dp[x] = dm[x] = 0.f;
                for (int j = 0; j < NQ; ++j) {
                    const float o = sDO[t * QP + j], y = sDU[t * QP + j];
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float u = sU[(sl + 8 * x) * QP + j];
                        dp[x] += o * u;
                        dm[x] -= y * u;
                    }
                }
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int s = sl + 8 * x;
                    if (s <= t) sdP[t * LP + s] += dp[x];
                    if (s < t) sdM[t * LP + s] += dm[x];
                }
            }
            // (e) owned (t, i): dO S0^T, -(beta Y) S0^T, U dS_C^T over this quarter's columns
            {
#pragma unroll 1
                for (int j = 0; j < NQ; j += 4) {
                    float4 s0v[4], dsv[4];
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const int i = ig + 32 * y;
                        s0v[y] = S0 ? __ldg(reinterpret_cast<const float4*>(S0 + (size_t)i * DV + j0 + j))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                        dsv[y] = __ldg(reinterpret_cast<const float4*>(dSC + (size_t)i * DV + j0 + j));
                    }
                    if (tg == 0) {
#pragma unroll
                        for (int y = 0; y < 4; ++y)
                            rowS[y] += s0v[y].x * dsv[y].x + s0v[y].y * dsv[y].y + s0v[y].z * dsv[y].z +
                                       s0v[y].w * dsv[y].w;
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int t = 4 * tg + x;
                        const float bt = sBeta[t];
                        const float o[4] = {sDO[t * QP + j], sDO[t * QP + j + 1], sDO[t * QP + j + 2], sDO[t * QP + j + 3]};
                        const float yy[4] = {bt * sDU[t * QP + j], bt * sDU[t * QP + j + 1], bt * sDU[t * QP + j + 2],
                                             bt * sDU[t * QP + j + 3]};
                        const float u[4] = {sU[t * QP + j], sU[t * QP + j + 1], sU[t * QP + j + 2], sU[t * QP + j + 3]};
#pragma unroll
                        for (int y = 0; y < 4; ++y) {
                            const float sv[4] = {s0v[y].x, s0v[y].y, s0v[y].z, s0v[y].w};
                            const float dv4[4] = {dsv[y].x, dsv[y].y, dsv[y].z, dsv[y].w};
#pragma unroll
                            for (int z = 0; z < 4; ++z) {
                                aQG[x][y] += o[z] * sv[z];
                                aKG[x][y] -= yy[z] * sv[z];
                                aKC[x][y] += u[z] * dv4[z];
                            }
                        }
                    }
                }
            }
            __syncthreads();  // the quarter buffers are rewritten next
        }

        // ---- P4: dbeta and dA = Diag(beta) dM
        if (tid < CH) {
            const int t = tid;
            float acc = sDb[t];
            for (int s = 0; s < t; ++s) acc += sdM[t * LP + s] * sA[t * LP + s];
            if (t < L) a.dbeta[(size_t)(t0 + t) * H + h] = acc;
            const float b = sBeta[t];
            for (int s = 0; s < t; ++s) sdM[t * LP + s] *= b;
        }
        // owned accumulators -> gradients of qb, k, g
        float dqb[4][4], dkk[4][4], dg[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int t = 4 * tg + x;
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int i = ig + 32 * y;
                float kv = 0.f, qv = 0.f;
                if (t < L) {
                    const size_t idx = ((size_t)(t0 + t) * H + h) * DK + i;
                    kv = ld_in(a.k, idx, a.in_bf16);
                    qv = a.scale * ld_in(a.q, idx, a.in_bf16);
                }
                const float g = sG[t * DK + i];
                const float gam = __expf(g), ec = __expf(sGC[i] - g);
                dqb[x][y] = gam * aQG[x][y];
                dkk[x][y] = gam * aKG[x][y] + ec * aKC[x][y];
                dg[x][y] = qv * gam * aQG[x][y] + kv * gam * aKG[x][y] - kv * ec * aKC[x][y];
                atomicAdd(&sDgC[i], kv * ec * aKC[x][y]);
            }
        }
        if (tg == 0) {
#pragma unroll
            for (int y = 0; y < 4; ++y) atomicAdd(&sDgC[ig + 32 * y], __expf(sGC[ig + 32 * y]) * rowS[y]);
        }
        __syncthreads();

        // ---- P5: the A / P contractions, block row by block row
        float* sC = sR;  // [3][16][128] contributions of the block's tokens (the quarter buffers are free)
        for (int bt = 0; bt < nb; ++bt) {
            build_factors(a, sF, sG, bt, t0, L, h, tid);
            __syncthreads();
            const int r = 16 * bt;
            {  // tokens t of the block, all threads: dKin_t = sum_s dA_ts Kout_s, dQin_t = sum_s dP_ts Kout_s
                const int tl = tid >> 5, i4 = (tid & 31) * 4, t = r + tl;
                if (t < L) {
                    float dki[4] = {0.f, 0.f, 0.f, 0.f}, dqi[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int s = 0; s <= t; ++s) {
                        const float wm = s < t ? sdM[t * LP + s] : 0.f, wp = sdP[t * LP + s];
                        const float4 ko = *reinterpret_cast<const float4*>(sF + s * FP + i4);
                        dki[0] += wm * ko.x; dki[1] += wm * ko.y; dki[2] += wm * ko.z; dki[3] += wm * ko.w;
                        dqi[0] += wp * ko.x; dqi[1] += wp * ko.y; dqi[2] += wp * ko.z; dqi[3] += wp * ko.w;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i4 + u;
                        const float e = __expf(sG[t * DK + i] - sG[r * DK + i]);
                        sC[(0 * 16 + tl) * DK + i] = e * dki[u];
                        sC[(1 * 16 + tl) * DK + i] = e * dqi[u];
                        sC[(2 * 16 + tl) * DK + i] = sF[(64 + tl) * FP + i] * dki[u] + sF[(80 + tl) * FP + i] * dqi[u];
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int t = 4 * tg + x;
                if ((t >> 4) == bt && t < L) {  // owner of a block token: take its contributions
                    const int tl = t - r;
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const int i = ig + 32 * y;
                        dkk[x][y] += sC[(0 * 16 + tl) * DK + i];
                        dqb[x][y] += sC[(1 * 16 + tl) * DK + i];
                        dg[x][y] += sC[(2 * 16 + tl) * DK + i];
                    }
                }
                if (t < r + 16 && t < L) {  // t as an earlier token s: dKout_t
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const int i = ig + 32 * y;
                        float dko = 0.f;
                        for (int tl = (t > r ? t - r : 0); tl < 16; ++tl) {
                            const int tt = r + tl;
                            if (tt >= L) break;
                            if (tt > t) dko += sdM[tt * LP + t] * sF[(64 + tl) * FP + i];
                            dko += sdP[tt * LP + t] * sF[(80 + tl) * FP + i];
                        }
                        const float e = __expf(sG[r * DK + i] - sG[t * DK + i]);
                        dkk[x][y] += e * dko;
                        dg[x][y] -= sF[t * FP + i] * dko;
                    }
                }
            }
            __syncthreads();
        }

        // ---- P6: dq, dk out; dg -> dlog_alpha (reverse cumulative sum over the chunk)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int t = 4 * tg + x;
            if (t < L) {
                const size_t base = ((size_t)(t0 + t) * H + h) * DK + ig;
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    a.dq[base + 32 * y] = a.scale * dqb[x][y];
                    a.dk[base + 32 * y] = dkk[x][y];
                }
            }
#pragma unroll
            for (int y = 0; y < 4; ++y) sF[t * FP + ig + 32 * y] = dg[x][y];
        }
        __syncthreads();
        if (tid < DK) {
            const int i = tid;
            float lv[CH];
#pragma unroll
            for (int t = 0; t < CH; ++t)
                lv[t] = t < L ? ld_in(a.log_alpha, ((size_t)(t0 + t) * H + h) * DK + i, a.in_bf16) : 0.f;
            float run = sDgC[i];  // g_C is g of the last token
#pragma unroll
            for (int t = CH - 1; t >= 0; --t) {
                if (t < L) {
                    run += sF[t * FP + i];
                    a.dla[((size_t)(t0 + t) * H + h) * DK + i] = lv[t] >= -5.f ? run : 0.f;
                }
            }
        }
        __syncthreads();  // shared memory is reused by the next item
    }
}

}  // namespace

size_t chunk_bwd_extra_bytes(int n_seqs, int H, int64_t max_seqlen) {
    const int64_t nck = (max_seqlen + CH - 1) / CH;
    const int64_t n_ckpt = max_seqlen / CH;
    return (size_t)n_seqs * H * STATE * sizeof(float) * (size_t)(nck + n_ckpt);
}

cudaError_t chunk_bwd_launch(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, const void* d_o, const float* d_final, float* dq, float* dk,
                             float* dv, float* dlog_alpha, float* dbeta, float* d_init, int B, int64_t T, int H,
                             const int32_t* cu, int n_seqs, int64_t max_seqlen, bool in_bf16, float scale,
                             void* workspace, size_t fwd_bytes, cudaStream_t stream) {
    static bool attr = false;
    static int sms = 0;
    cudaError_t err;
    if (!attr) {
        if ((err = cudaFuncSetAttribute(chain_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CB_SMEM)) !=
                cudaSuccess ||
            (err = cudaFuncSetAttribute(bwd_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BI_SMEM)) !=
                cudaSuccess)
            return err;
        int dev = 0;
        if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
        if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
        attr = true;
    }
    const int N = cu ? n_seqs : B;
    const int64_t maxlen = cu ? max_seqlen : T;
    const int nck = (int)((maxlen + CH - 1) / CH);
    const int n_ckpt = (int)(maxlen / CH);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    float* ckpt = reinterpret_cast<float*>(ws + fwd_bytes);
    float* ds_end = ckpt + (size_t)N * n_ckpt * H * STATE;
    // 1. the forward walk again, without outputs: chunk slots and chunk-boundary states
    err = chunk_fwd_launch(q, k, v, log_alpha, beta, init_state, nullptr, nullptr, B, T, H, cu, n_seqs, max_seqlen,
                           in_bf16, false, scale, nullptr, nullptr, 0.f, n_ckpt > 0 ? ckpt : nullptr, CH, 1, KCP_NONE,
                           nullptr, workspace, fwd_bytes, stream, nullptr, nullptr);
    if (err != cudaSuccess) return err;
    // the forward's slot region (whole-sequence workspace: one pass)
    const size_t head = (chunk_fixed_bytes(N, H, true) + 1023) & ~(size_t)1023;
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.d_o = d_o;
    a.init_state = init_state; a.d_final = d_final; a.d_init = d_init;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dla = dlog_alpha; a.dbeta = dbeta;
    a.cu = cu;
    a.slots = ws + head;
    a.ckpt = ckpt;
    a.ds_end = ds_end;
    a.status = reinterpret_cast<uint32_t*>(ws);
    a.T = T; a.H = H; a.n_seqs = N; a.wc = nck > 0 ? nck : 1; a.n_ckpt = n_ckpt;
    a.scale = scale;
    a.in_bf16 = in_bf16 ? 1 : 0;
    // 2. the reverse walk: dL/d(state) at every chunk end, dL/dS_0
    prof_begin(PROF_CHAIN_BWD, stream);
    chain_bwd_kernel<<<dim3(NSL, H, N), CB_THREADS, CB_SMEM, stream>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    prof_end(PROF_CHAIN_BWD, stream);
    // 3. the chunk-local gradients
    const int64_t n_items = (int64_t)N * a.wc * H;
    if (nck > 0 && n_items > 0) {
        const unsigned grid = (unsigned)(n_items < sms ? n_items : sms);
        prof_begin(PROF_INTRA_BWD, stream);
        bwd_intra_kernel<<<grid, BI_THREADS, BI_SMEM, stream>>>(a, n_items);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        prof_end(PROF_INTRA_BWD, stream);
    }
    return cudaSuccess;
}

}  // namespace kda
