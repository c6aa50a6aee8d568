// kda_bwd.cu -- backward pass of the chunkwise KDA prefill.
//
// The pages describe no backward pass.  This is the exact gradient of the
// forward (the recurrence and its chunkwise form: K3 article summaries,
// xhh.club tag page, items "KDA recurrence form" and "chunkwise parallel
// algorithm"), arranged chunkwise:
//   1. the forward walk is recomputed without outputs; it leaves every chunk's
//      slot (M_lr, Q', Gamma_C) in the workspace and the state at every chunk
//      boundary in a checkpoint buffer;
//   2. chain_bwd_tc_kernel walks the chunks of a sequence in reverse with
//      dS = dL/d(state at the end of chunk c):
//          dS_end[c] = dS,    dS <- Diag(Gamma_C) dS - M_lr^T dS + Q'^T dO_c
//      starting from dL/dS_final and ending with dL/dS_0;
//   3. bwd_tc_kernel takes one (chunk, head) at a time, with the chunk-start
//      state S0 and dS_C = dS_end[c], and forms dq, dk, dv, dbeta, dlog_alpha of
//      the chunk's tokens; its products run on the tensor cores.
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
// The A / P terms use the forward's per-16-token-tile exponent references G_b (g
// just before tile b): e^{g_t - g_s} = e^{g_t - G_b} e^{G_b - g_s}, so no operand
// overflows.  Products run on the tensor cores with bf16 operands and fp32
// accumulators; M^-1, the exponentials and the gradient assembly are fp32.
#include <string.h>

#include "kda_launch.h"
#include "kda_profile.h"
#include "kda_slots.h"
#include "kda_sm100.cuh"
#include "kda_tri.cuh"

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
    const uint8_t* ckpt;       // states after every whole chunk, bf16 images [n_seqs][n_ckpt][H]
    uint8_t* ds_end;           // dL/d(state at chunk end), bf16 images [n_seqs][wc][H]
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

constexpr int BT_THREADS = 512;  // threads of the chunk-local kernel

// Pulls an item's token rows (q, k, v, log_alpha, dO: 64 rows each), its
// chunk-start state and its end-of-chunk state gradient into L2 ahead of use.
// (sequence, chunk, head) of an item: item = (n * wc + chunk) * H + h (items < 2^31)
KDA_DEV void bwd_item(const BwdArgs& a, int64_t item, int& n, int& c, int& h) {
    const uint32_t it = (uint32_t)item, rest = it / (uint32_t)a.H;
    h = (int)(it - rest * (uint32_t)a.H);
    const uint32_t nn = rest / (uint32_t)a.wc;
    c = (int)(rest - nn * (uint32_t)a.wc);
    n = (int)nn;
}

template <bool IN_BF16>
KDA_DEV void prefetch_item(const BwdArgs& a, int64_t item, int64_t n_items, int tid) {
    if (item >= n_items) return;
    const int H = a.H;
    int n, c, h;
    bwd_item(a, item, n, c, h);
    int64_t s_beg, s_end;
    bwd_seq_range(a, n, s_beg, s_end);
    const int64_t t0 = s_beg + (int64_t)c * CH;
    if (t0 >= s_end) return;
    const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
    constexpr size_t row = DK * (IN_BF16 ? 2 : 4);  // bytes of one head row
    constexpr int lines_row = (int)(row / 128);
    const void* tens[5] = {a.q, a.k, a.v, a.log_alpha, a.d_o};
    for (int e = tid; e < 5 * CH * lines_row; e += BT_THREADS) {
        const int tsr = e / (CH * lines_row), rem = e % (CH * lines_row), t = rem / lines_row, ln = rem % lines_row;
        if (t >= L) continue;
        const char* p = reinterpret_cast<const char*>(tens[tsr]) + ((size_t)(t0 + t) * H + h) * row + ln * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
    }
    const char* S0 = c == 0 ? reinterpret_cast<const char*>(a.init_state ? a.init_state + ((size_t)n * H + h) * STATE
                                                                            : nullptr)
                            : reinterpret_cast<const char*>(a.ckpt + (((size_t)n * a.n_ckpt + (c - 1)) * H + h) *
                                                                         STATE_IMG_BYTES);
    const uint32_t s0_bytes = c == 0 ? STATE * 4 : STATE_IMG_BYTES;
    const char* dSC = reinterpret_cast<const char*>(a.ds_end + (((size_t)n * a.wc + c) * H + h) * STATE_IMG_BYTES);
    for (uint32_t e = tid; e < (s0_bytes + STATE_IMG_BYTES) / 128; e += BT_THREADS) {
        const char* p = e < s0_bytes / 128 ? (S0 ? S0 + (size_t)e * 128 : nullptr) : dSC + (size_t)(e - s0_bytes / 128) * 128;
        if (p) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
    }
}

// ------------------------------------------------ chunk-local part (tensor cores)
// One item = (chunk, head); 512 threads, thread (c = tid % 128, q4 = tid / 128) owns
// channel c (key channel i, or value column j) and the 16-token tile q4.  Every product
// of the item runs on the tensor cores (tcgen05.mma kind::f16: bf16 operand images in
// shared memory, fp32 accumulators in TMEM); the SIMT phases between them build the
// operand images, invert M in fp32 and assemble the gradients.
//
// Operand images: row-major with 16-byte pieces along the columns, no swizzle:
// element (r, c) of an image with nc columns at il_off(r, c, nc).  The same image is a
// K-major operand (columns = K) or an MN-major one (columns = M or N), which is how each
// image below serves two products.  Transposed products keep a channel (i or j) in the
// 128 TMEM lanes, so thread (c, q4) reads its own channel's row.
//   I1 KQr  [i][t']  t' < 64: k_t e^{g_t - G_b},  t' >= 64: scale q_t e^{g_t - G_b}  (b = tile of t)
//   I2 KC   [i][sv]  the 160 column versions of the keys (forward stage 1): sv < 64:
//                    k_s e^{G_b(s) - g_s}; Kb1/Kb2/Kb3: tiles before b w.r.t. G_b
//   I3 KG   [i][t]   k_t e^{g_t};   I4 KCe [i][t]  k_t e^{g_C - g_t}
//   I5 S0   [i][j];  I6 dSC [i][j]  (chunk-start state, gradient at the chunk end)
//   I7 [Y|dO] [j][t'] t' < 64: Y_t, t' >= 64: dO_t
//   I8 P    [t][s];  I9 Minv [t][s];  I10 beta R^T [j][s];  I11 dU^T [j][s];  I12 U^T [j][t]
//   I13 [A'|P'] [t'][sv]  dA (rows < 64) and dP (rows >= 64) placed at the column version
//                    their row's tile uses, zero elsewhere
// Products (M x N x K, D in TMEM with lane = M row):
//   stage 1  A/P raw = I1^T-rows x I2            128 x 160 x 128   (as the forward)
//            X1^T = S0^T (K o Gam)^T              128 x  64 x 128   (R = V - (K o Gam) S0)
//            dU^T = dSC^T K^C^T                   128 x  64 x 128
//   stage 2  U^T = (beta R)^T Minv^T              128 x  64 x  64
//            dU^T += dO^T P                       128 x  64 x  64
//   stage 3  Y^T = dU^T Minv                      128 x  64 x  64
//            aKC = dSC U^T  [i][t]                128 x  64 x 128
//   stage 4  [-dM ; dP] = [Y ; dO] U^T            128 x  64 x 128
//            [S0 Y^T | S0 dO^T]  [i][t']          128 x 128 x 128
//   stage 5  [RowA | RowP]^T = KC^T-cols x [A';P'] 128 x 128 x 160
//            Col^T = KQr x [A';P']                128 x 160 x 128
// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t BT_I5 = 0, BT_I6 = 32768, BT_I7 = 65536;
constexpr uint32_t BT_I1 = 98304, BT_I2 = 131072;                       // stage-1 copies
constexpr uint32_t BT_N = 98304, BT_X = BT_N + 17408, BT_TMP = BT_X + 17408;  // inverse (fp32)
constexpr uint32_t BT_I8 = BT_TMP + 8192, BT_I9 = BT_I8 + 8192, BT_I10 = BT_I9 + 8192, BT_I11 = BT_I10;
constexpr uint32_t BT_I12 = 98304;
constexpr uint32_t BT_I3 = BT_I10 + 16384, BT_I4 = BT_I3 + 16384;
constexpr uint32_t BT_I13 = 0, BT_I1B = 40960, BT_I2B = 73728;          // stage-5 images
constexpr uint32_t BT_I2L = 114688, BT_I1L = 155648;                    // their low parts
constexpr uint32_t BT_MISC = BT_I4 + 16384;
constexpr uint32_t BT_BETA = BT_MISC, BT_G = BT_BETA + 256, BT_TOT = BT_G + 2560, BT_RS = BT_TOT + 2048,
                   BT_DGC = BT_RS + 2048, BT_DB = BT_DGC + 2048, BT_BAR = BT_DB + 256, BT_TPTR = BT_BAR + 64;
static_assert(8 * 8 <= 64, "barriers");
constexpr uint32_t BT_SMEM = BT_TPTR + 16 + 1024;
constexpr int BT_LDA = TRI_LDA;
// TMEM columns
constexpr uint32_t TB_AP = 0, TB_X1 = 160, TB_DU = 224, TB_U = 288, TB_Y = 352, TB_KC = 416;
constexpr uint32_t TB_S4A = 288, TB_S4B = 160, TB_S5A = 288, TB_S5B = 0;
// column versions of the keys (forward stage 1): Kd [0,64), Kb1 [64,80), Kb2 [80,112), Kb3 [112,160)
constexpr uint32_t SV_B1 = 64, SV_B2 = 80, SV_B3 = 112, NSV = 160;

static_assert(BT_I10 + 16384 <= BT_I3, "I10 overlaps I3");
static_assert(BT_I2 + 40960 <= BT_I3, "stage-1 KC image overlaps KG");
static_assert(BT_TMP + 8192 <= BT_I8, "inverse scratch overlaps P");
static_assert(BT_SMEM <= 227 * 1024, "shared memory");
static_assert(BT_I1L + 32768 <= BT_MISC, "stage-5 low parts overlap the scalars");

KDA_DEV uint32_t il_off(uint32_t r, uint32_t c, uint32_t nc) {
    return (r >> 3) * (16u * nc) + (c >> 3) * 128u + (r & 7u) * 16u + (c & 7u) * 2u;
}
// descriptor of an image with nc columns read with its columns as the MN dimension
// (rows = K) or as the K dimension (rows = M/N); `col0` selects a first column (multiple of 8)
KDA_DEV uint64_t desc_mn(uint32_t addr, uint32_t nc, uint32_t col0 = 0) {
    return sdesc_interleave(addr + (col0 >> 3) * 128u, 16u * nc, 128u);
}
KDA_DEV uint64_t desc_k(uint32_t addr, uint32_t nc, uint32_t col0 = 0) {
    return sdesc_interleave(addr + (col0 >> 3) * 128u, 128u, 16u * nc);
}
// K-step (16) advance of the two views, in bytes
KDA_DEV constexpr uint32_t step_mn(uint32_t nc) { return 32u * nc; }
constexpr uint32_t STEP_K = 256u;

// D (+)= A B^T over nk steps of K = 16
KDA_DEV void mma_run(uint32_t d, uint64_t ad, uint32_t astep, uint64_t bd, uint32_t bstep, uint32_t idesc, int nk,
                     bool acc) {
    for (int kk = 0; kk < nk; ++kk)
        mma_bf16(d, ad + ((uint32_t)kk * astep >> 4), bd + ((uint32_t)kk * bstep >> 4), idesc,
                 (acc || kk > 0) ? 1u : 0u);
}

KDA_DEV void tmem_ld8(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}

KDA_DEV uint4 pack8f(const float* x) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
}
KDA_DEV float lo_bf(uint32_t w) { return __uint_as_float(w << 16); }
KDA_DEV float hi_bf(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
KDA_DEV void st16(uint8_t* p, const float* x) { *reinterpret_cast<uint4*>(p) = pack8f(x); }
// x as the sum of two bf16 images, hi = bf16(x) and lo = bf16(x - hi): a product with
// both (two MMAs into one accumulator) carries about 16 bits of x instead of 8
KDA_DEV void st16_hilo(uint8_t* hi, uint8_t* lo, const float* x) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hw[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);  // the high parts, rounded to nearest
        lw[e] = pack_bf16x2(x[2 * e] - lo_bf(hw[e]), x[2 * e + 1] - hi_bf(hw[e]));
    }
    *reinterpret_cast<uint4*>(hi) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(lo) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}
KDA_DEV void st16z(uint8_t* p) { *reinterpret_cast<uint4*>(p) = make_uint4(0u, 0u, 0u, 0u); }

// Sum over the 32 lanes of v[u] for each u < 16; lane l ends with the sum for token
// u = l >> 1 (both lanes of a pair hold it).  16 shuffles.
KDA_DEV float lane_sum16(float (&v)[16], int lane) {
    float w8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool up = lane & 16;
        const float send = up ? v[k] : v[k + 8], keep = up ? v[k + 8] : v[k];
        w8[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 16);
    }
    float w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const bool up = lane & 8;
        const float send = up ? w8[k] : w8[k + 4], keep = up ? w8[k + 4] : w8[k];
        w4[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 8);
    }
    float w2[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const bool up = lane & 4;
        const float send = up ? w4[k] : w4[k + 2], keep = up ? w4[k + 2] : w4[k];
        w2[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 4);
    }
    const bool up = lane & 2;
    float w1 = (up ? w2[1] : w2[0]) + __shfl_xor_sync(0xFFFFFFFFu, up ? w2[0] : w2[1], 2);
    w1 += __shfl_xor_sync(0xFFFFFFFFu, w1, 1);
    return w1;  // token index: 8 (lane>>4 & 1) + 4 (lane>>3 & 1) + 2 (lane>>2 & 1) + (lane>>1 & 1)
}
KDA_DEV int lane_sum16_token(int lane) { return (lane >> 1) & 15; }

// log-decays of the 16 tokens of tile q4 at channel c: per-step decays and the in-tile
// prefix / suffix products E1 = e^{g_t - G_q4}, E3 = e^{G_{q4+1} - g_t}; returns the tile total
template <bool IN_BF16>
KDA_DEV float tile_decays(const BwdArgs& a, size_t base_c, size_t rowk, int q4, int L, float (&E1)[16],
                          float (&E3)[16], uint32_t* keep_mask) {
    float alpha[16];
    float run = 0.f;
    uint32_t keep = 0;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int t = 16 * q4 + u;
        float l = 0.f;
        if (t < L) {
            l = ld_in(a.log_alpha, base_c + (size_t)t * rowk, IN_BF16 ? 1 : 0);
            if (l >= -5.f) keep |= 1u << u;
            l = fmaxf(l, -5.f);
        }
        run += l;
        alpha[u] = __expf(l);
    }
    E1[0] = alpha[0];
#pragma unroll
    for (int u = 1; u < 16; ++u) E1[u] = E1[u - 1] * alpha[u];
    E3[15] = 1.f;
#pragma unroll
    for (int u = 14; u >= 0; --u) E3[u] = E3[u + 1] * alpha[u + 1];
    if (keep_mask) *keep_mask = keep;
    return run;
}

// the item's raw tiles (bf16 inputs): [64 tokens][128 channels] each, by TMA, at the start
// of the item into the region of the state images (written after the tiles are read)
struct BwdMaps {
    CUtensorMap la, k, q, v, d_o;
};
constexpr uint32_t BT_RLA = 0, BT_RK = 16384, BT_RQ = 32768, BT_RV = 49152, BT_RDO = 65536;

KDA_DEV float raw_bf16(const uint8_t* sm, uint32_t tile, int t, int c, int L) {
    return t < L ? __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(sm + tile + (uint32_t)(t * 128 + c) * 2u)
                                   << 16)
                 : 0.f;
}

template <bool IN_BF16>
__global__ void __launch_bounds__(BT_THREADS, 1) bwd_tc_kernel(const BwdArgs a, const __grid_constant__ BwdMaps maps,
                                                            int64_t n_items) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = tid & 127, q4 = tid >> 7, qd = warp & 3;
    const int H = a.H;
    float* s_beta = reinterpret_cast<float*>(sm + BT_BETA);
    float* s_G = reinterpret_cast<float*>(sm + BT_G);       // [5][128]
    float* s_tot = reinterpret_cast<float*>(sm + BT_TOT);   // [4][128]
    float* s_rs = reinterpret_cast<float*>(sm + BT_RS);     // [4][128] rowsum(S0 o dSC) partials
    float* s_dgc = reinterpret_cast<float*>(sm + BT_DGC);   // [4][128] dL/dg_C partials
    float* s_db = reinterpret_cast<float*>(sm + BT_DB);     // [64] dL/dbeta
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BT_BAR);  // [6]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + BT_TPTR);
    if (warp == 0) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&bar[i], 1);  // 0-5: the stages' products, 6: raw tiles, 7: states
        fence_mbar_init();
        if constexpr (IN_BF16) {
            prefetch_tmap(&maps.la);
            prefetch_tmap(&maps.k);
            prefetch_tmap(&maps.q);
            prefetch_tmap(&maps.v);
            prefetch_tmap(&maps.d_o);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;
    const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
    uint32_t par = 0;
    bool failed = false;
    int committed = 0;  // barriers committed in the current item (for the bounded drain)

    // waits for the tensor-core products of barrier i; a wait that gives up ends the
    // kernel's work on every thread at once
    auto wait_mma = [&](int i) -> bool {
        const bool ok = mbar_wait(&bar[i], par, a.status);
        const bool any_fail = __syncthreads_or(!ok);
        tc_fence_after();
        return !any_fail;
    };
    auto images_ready = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    for (int64_t item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
        int n, cidx, h;
        bwd_item(a, item, n, cidx, h);
        int64_t s_beg, s_end;
        bwd_seq_range(a, n, s_beg, s_end);
        const int64_t t0 = s_beg + (int64_t)cidx * CH;
        if (t0 >= s_end) continue;  // uniform over the CTA
        const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);
        // the chunk-start state: the initial state (fp32, or none) for the first chunk, else the
        // forward walk's bf16 image; the chunk-end state gradient: the reverse walk's bf16 image
        const float* S0f = (cidx == 0 && a.init_state) ? a.init_state + ((size_t)n * H + h) * STATE : nullptr;
        const uint8_t* S0img = cidx == 0 ? nullptr : a.ckpt + (((size_t)n * a.n_ckpt + (cidx - 1)) * H + h) * STATE_IMG_BYTES;
        const uint8_t* dSCimg = a.ds_end + (((size_t)n * a.wc + cidx) * H + h) * STATE_IMG_BYTES;
        prefetch_item<IN_BF16>(a, item + gridDim.x, n_items, tid);
        const size_t rowk = (size_t)H * DK;
        const size_t base_c = ((size_t)t0 * H + h) * DK + c;  // (token t0, head h, channel c)
        const int ib = IN_BF16 ? 1 : 0;

        // ================================================================ phase A
        if constexpr (IN_BF16) {
            if (tid == 0) {
                fence_async_smem();  // the previous item's generic reads of this region are done
                mbar_arrive_expect_tx(&bar[6], 5u * 16384u);
                tma_load_2d(sm + BT_RLA, &maps.la, h * DK, (int)t0, &bar[6]);
                tma_load_2d(sm + BT_RK, &maps.k, h * DK, (int)t0, &bar[6]);
                tma_load_2d(sm + BT_RQ, &maps.q, h * DK, (int)t0, &bar[6]);
                tma_load_2d(sm + BT_RV, &maps.v, h * DV, (int)t0, &bar[6]);
                tma_load_2d(sm + BT_RDO, &maps.d_o, h * DV, (int)t0, &bar[6]);
            }
            committed = 7;  // for the drain: the tile loads are in flight
            if (!wait_mma(6)) { failed = true; break; }
            committed = 0;
        }
        float E1[16], E3[16];
        float run;
        uint32_t lar2[8];      // raw log-decays of this thread's tokens (bf16 pairs), for phases E and F
        uint32_t keep_la = 0;  // tokens whose log-decay is at or above the floor (the clamp passes them)
        if constexpr (IN_BF16) {
            float alpha[16];
            run = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = 16 * q4 + u;
                const float raw = raw_bf16(sm, BT_RLA, t, c, L);
                if (u & 1) lar2[u >> 1] |= __float_as_uint(raw) & 0xFFFF0000u;
                else lar2[u >> 1] = __float_as_uint(raw) >> 16;
                if (t < L && raw >= -5.f) keep_la |= 1u << u;
                const float l = t < L ? fmaxf(raw, -5.f) : 0.f;
                run += l;
                alpha[u] = __expf(l);
            }
            E1[0] = alpha[0];
#pragma unroll
            for (int u = 1; u < 16; ++u) E1[u] = E1[u - 1] * alpha[u];
            E3[15] = 1.f;
#pragma unroll
            for (int u = 14; u >= 0; --u) E3[u] = E3[u + 1] * alpha[u + 1];
        } else {
            run = tile_decays<IN_BF16>(a, base_c, rowk, q4, L, E1, E3, nullptr);
        }
        s_tot[q4 * 128 + c] = run;
        if (tid < CH) {
            s_beta[tid] = tid < L ? ld_in(a.beta, (size_t)(t0 + tid) * H + h, ib) : 0.f;
            s_db[tid] = 0.f;
        }
        __syncthreads();
        {
            float off = 0.f;
#pragma unroll
            for (int qq = 0; qq < 3; ++qq)
                if (qq < q4) off += s_tot[qq * 128 + c];
            s_G[(q4 + 1) * 128 + c] = off + run;
            if (q4 == 0) s_G[c] = 0.f;
        }
        __syncthreads();
        float G[5];
#pragma unroll
        for (int b = 0; b < 5; ++b) G[b] = s_G[b * 128 + c];
        const float Gs = (q4 == 0) ? G[0] : (q4 == 1) ? G[1] : (q4 == 2) ? G[2] : G[3];
        const float Gn = (q4 == 0) ? G[1] : (q4 == 1) ? G[2] : (q4 == 2) ? G[3] : G[4];
        // raw k, q, v of this thread's 16 tokens (bf16 bit pairs; exact for bf16 inputs)
        uint32_t kr2[8], qr2[8], vr2[8], dor2[8];
        {
            const float eD = __expf(Gs - Gn);
            const float f2 = __expf(((q4 == 0) ? G[2] : G[3]) - Gn);
            const float f3 = __expf(G[3] - Gn);
            const float eG = __expf(Gs), eC = __expf(G[4] - Gn);
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int tf = 16 * q4 + 8 * m;
                float kv[8], qv[8], vv[8], dov[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = tf + e;
                    if constexpr (IN_BF16) {
                        kv[e] = raw_bf16(sm, BT_RK, t, c, L);
                        qv[e] = raw_bf16(sm, BT_RQ, t, c, L);
                        vv[e] = raw_bf16(sm, BT_RV, t, c, L);
                        dov[e] = raw_bf16(sm, BT_RDO, t, c, L);
                    } else {
                        const bool in = t < L;
                        const size_t idx = base_c + (size_t)t * rowk;
                        kv[e] = in ? ld_in(a.k, idx, ib) : 0.f;
                        qv[e] = in ? ld_in(a.q, idx, ib) : 0.f;
                        vv[e] = in ? ld_in(a.v, idx, ib) : 0.f;
                        dov[e] = in ? ld_in(a.d_o, idx, ib) : 0.f;
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    kr2[(8 * m + e) >> 1] = pack_bf16x2(kv[e], kv[e + 1]);
                    qr2[(8 * m + e) >> 1] = pack_bf16x2(qv[e], qv[e + 1]);
                    vr2[(8 * m + e) >> 1] = pack_bf16x2(vv[e], vv[e + 1]);
                    dor2[(8 * m + e) >> 1] = pack_bf16x2(dov[e], dov[e + 1]);
                }
                float x[8], y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = kv[e] * E1[8 * m + e];
                    y[e] = qv[e] * E1[8 * m + e] * a.scale;
                }
                st16(sm + BT_I1 + il_off(c, tf, 128), x);
                st16(sm + BT_I1 + il_off(c, 64 + tf, 128), y);
                float k3[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    k3[e] = kv[e] * E3[8 * m + e];
                    x[e] = k3[e] * eD;
                }
                st16(sm + BT_I2 + il_off(c, tf, NSV), x);
                if (q4 == 0) {
                    st16(sm + BT_I2 + il_off(c, SV_B1 + tf, NSV), k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f2;
                    st16(sm + BT_I2 + il_off(c, SV_B2 + tf, NSV), x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f3;
                    st16(sm + BT_I2 + il_off(c, SV_B3 + tf, NSV), x);
                } else if (q4 == 1) {
                    st16(sm + BT_I2 + il_off(c, SV_B2 + tf, NSV), k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f3;
                    st16(sm + BT_I2 + il_off(c, SV_B3 + tf, NSV), x);
                } else if (q4 == 2) {
                    st16(sm + BT_I2 + il_off(c, SV_B3 + tf, NSV), k3);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = kv[e] * E1[8 * m + e] * eG;  // k e^{g}
                    y[e] = k3[e] * eC;                  // k e^{g_C - g}
                }
                st16(sm + BT_I3 + il_off(c, tf, 64), x);
                st16(sm + BT_I4 + il_off(c, tf, 64), y);
            }
            __syncthreads();  // every read of the raw tiles is done: their region takes S0, dSC, dO^T
#pragma unroll
            for (int m = 0; m < 2; ++m)  // dO^T: row j = c
                *reinterpret_cast<uint4*>(sm + BT_I7 + il_off(c, 64 + 16 * q4 + 8 * m, 128)) =
                    make_uint4(dor2[4 * m], dor2[4 * m + 1], dor2[4 * m + 2], dor2[4 * m + 3]);
            // S0 and dSC: the images arrive by bulk copies into the region the raw tiles just left
            // (the first chunk's S0 comes from the fp32 initial state, converted here)
            if (tid == 0) {
                fence_async_smem();
                mbar_arrive_expect_tx(&bar[7], S0img ? 2u * STATE_IMG_BYTES : STATE_IMG_BYTES);
                if (S0img) bulk_g2s(sm + BT_I5, S0img, STATE_IMG_BYTES, &bar[7]);
                bulk_g2s(sm + BT_I6, dSCimg, STATE_IMG_BYTES, &bar[7]);
            }
            if (!S0img) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int j = 32 * q4 + 8 * m;
                    float s8[8];
                    if (S0f) {
                        const float4 u0 = __ldg(reinterpret_cast<const float4*>(S0f + (size_t)c * DV + j));
                        const float4 u1 = __ldg(reinterpret_cast<const float4*>(S0f + (size_t)c * DV + j + 4));
                        s8[0] = u0.x; s8[1] = u0.y; s8[2] = u0.z; s8[3] = u0.w;
                        s8[4] = u1.x; s8[5] = u1.y; s8[6] = u1.z; s8[7] = u1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) s8[e] = 0.f;
                    }
                    st16(sm + BT_I5 + il_off(c, j, 128), s8);
                }
            }
            committed = 8;  // for the drain: the state copies are in flight
            if (!wait_mma(7)) { failed = true; break; }
            committed = 0;
            // rowsum(S0 o dSC) of row c over columns [32 q4, 32 q4 + 32), from the images
            float rs = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t off = il_off(c, 32 * q4 + 8 * m, 128);
                const uint4 x = *reinterpret_cast<const uint4*>(sm + BT_I5 + off);
                const uint4 y = *reinterpret_cast<const uint4*>(sm + BT_I6 + off);
                const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) rs += lo_bf(xs[e]) * lo_bf(ys[e]) + hi_bf(xs[e]) * hi_bf(ys[e]);
            }
            s_rs[q4 * 128 + c] = rs;
        }
        images_ready();

        // ------------------------------------------------------------- stage 1
        if (tid == 0) {
            mma_run(tm + TB_AP, desc_mn(sb + BT_I1, 128), step_mn(128), desc_mn(sb + BT_I2, NSV), step_mn(NSV),
                    idesc_bf16_major(128, 160, 1, 1), 8, false);
            mma_commit(&bar[0]);
            mma_run(tm + TB_X1, desc_mn(sb + BT_I5, 128), step_mn(128), desc_mn(sb + BT_I3, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 1, 1), 8, false);
            mma_run(tm + TB_DU, desc_mn(sb + BT_I6, 128), step_mn(128), desc_mn(sb + BT_I4, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 1, 1), 8, false);
            mma_commit(&bar[1]);
        }
        committed = 2;

        // ================================================================ phase B
        if (!wait_mma(0)) { failed = true; break; }
        {   // A (rows 0..63) -> N = Diag(beta) A fp32;  P (rows 64..127) -> image I8 [t][s]
            float* sN = reinterpret_cast<float*>(sm + BT_N);
            const int p = q4, r = 32 * qd + lane;
            const bool isP = r >= 64;
            const int t = r & 63, bt = t >> 4;
            float dA[16], dB[16], dC[16];
            tmem_ld16(lane_addr + TB_AP + 16 * p, dA);
            if ((qd & 1) == 0) {
                if (p == 0) tmem_ld16(lane_addr + TB_AP + SV_B1, dB);
            } else {
                if (p < 2) tmem_ld16(lane_addr + TB_AP + SV_B2 + 16 * p, dB);
                if (p < 3) tmem_ld16(lane_addr + TB_AP + SV_B3 + 16 * p, dC);
            }
            tmem_ld_wait();
            float d[16];
            if (p >= bt) {
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) {
                    const int s = 16 * p + s16;
                    const bool keep = (p == bt) && (isP ? (s <= t) : (s < t));
                    d[s16] = keep ? dA[s16] : 0.f;
                }
            } else if (bt == 3) {
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) d[s16] = dC[s16];
            } else {
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) d[s16] = dB[s16];
            }
            if (isP) {
                st16(sm + BT_I8 + il_off(t, 16 * p, 64), d);
                st16(sm + BT_I8 + il_off(t, 16 * p + 8, 64), d + 8);
            } else {
                const float bt_ = s_beta[t];
                float4* dst = reinterpret_cast<float4*>(sN + t * BT_LDA + 16 * p);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(bt_ * d[4 * i], bt_ * d[4 * i + 1], bt_ * d[4 * i + 2], bt_ * d[4 * i + 3]);
            }
        }
        if (!wait_mma(1)) { failed = true; break; }
        float R[16];
        {   // R = V - (K o Gam) S0 for this thread's value column j = c and 16 tokens
            float x1[16];
            tmem_ld16(lane_addr + TB_X1 + 16 * q4, x1);
            tmem_ld_wait();
            float br[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float vv = IN_BF16 ? ((u & 1) ? hi_bf(vr2[u >> 1]) : lo_bf(vr2[u >> 1]))
                                         : (16 * q4 + u < L ? ld_in(a.v, base_c + (size_t)(16 * q4 + u) * rowk, 0) : 0.f);
                R[u] = vv - x1[u];
                br[u] = s_beta[16 * q4 + u] * R[u];
            }
            st16(sm + BT_I10 + il_off(c, 16 * q4, 64), br);
            st16(sm + BT_I10 + il_off(c, 16 * q4 + 8, 64), br + 8);
        }
        __syncthreads();
        tri_inverse64(reinterpret_cast<const float*>(sm + BT_N), reinterpret_cast<float*>(sm + BT_X),
                      reinterpret_cast<float*>(sm + BT_TMP), reinterpret_cast<float*>(sm + BT_N), tid);
        {   // Minv image I9 [t][s] (blocks above the diagonal are zero)
            const float* sX = reinterpret_cast<const float*>(sm + BT_X);
            const float* sP = reinterpret_cast<const float*>(sm + BT_N);  // second half of the lower-left sums
            const int t = tid >> 3, s0 = (tid & 7) * 8;
            float v8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if ((s0 >> 4) <= (t >> 4)) {
                float4 x0 = *reinterpret_cast<const float4*>(sX + t * BT_LDA + s0);
                float4 x1 = *reinterpret_cast<const float4*>(sX + t * BT_LDA + s0 + 4);
                if (t >= 48 && s0 < 32) {
                    const float4 p0 = *reinterpret_cast<const float4*>(sP + (t - 48) * 32 + s0);
                    const float4 p1 = *reinterpret_cast<const float4*>(sP + (t - 48) * 32 + s0 + 4);
                    x0.x += p0.x; x0.y += p0.y; x0.z += p0.z; x0.w += p0.w;
                    x1.x += p1.x; x1.y += p1.y; x1.z += p1.z; x1.w += p1.w;
                }
                v8[0] = x0.x; v8[1] = x0.y; v8[2] = x0.z; v8[3] = x0.w;
                v8[4] = x1.x; v8[5] = x1.y; v8[6] = x1.z; v8[7] = x1.w;
            }
            st16(sm + BT_I9 + il_off(t, s0, 64), v8);
        }
        images_ready();

        // ------------------------------------------------------------- stage 2
        if (tid == 0) {
            mma_run(tm + TB_U, desc_k(sb + BT_I10, 64), STEP_K, desc_k(sb + BT_I9, 64), STEP_K,
                    idesc_bf16_major(128, 64, 0, 0), 4, false);
            mma_run(tm + TB_DU, desc_k(sb + BT_I7, 128, 64), STEP_K, desc_mn(sb + BT_I8, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 0, 1), 4, true);
            mma_commit(&bar[2]);
        }
        committed = 3;

        // ================================================================ phase C
        if (!wait_mma(2)) { failed = true; break; }
        {
            float x[16];
            tmem_ld16(lane_addr + TB_U + 16 * q4, x);
            tmem_ld_wait();
            st16(sm + BT_I12 + il_off(c, 16 * q4, 64), x);
            st16(sm + BT_I12 + il_off(c, 16 * q4 + 8, 64), x + 8);
            tmem_ld16(lane_addr + TB_DU + 16 * q4, x);
            tmem_ld_wait();
            st16(sm + BT_I11 + il_off(c, 16 * q4, 64), x);
            st16(sm + BT_I11 + il_off(c, 16 * q4 + 8, 64), x + 8);
        }
        images_ready();

        // ------------------------------------------------------------- stage 3
        if (tid == 0) {
            mma_run(tm + TB_Y, desc_k(sb + BT_I11, 64), STEP_K, desc_mn(sb + BT_I9, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 0, 1), 4, false);
            mma_run(tm + TB_KC, desc_k(sb + BT_I6, 128), STEP_K, desc_mn(sb + BT_I12, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 0, 1), 8, false);
            mma_commit(&bar[3]);
        }
        committed = 4;

        // ================================================================ phase D
        if (!wait_mma(3)) { failed = true; break; }
        {
            float y[16];
            tmem_ld16(lane_addr + TB_Y + 16 * q4, y);
            tmem_ld_wait();
            float pr[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = 16 * q4 + u;
                pr[u] = y[u] * R[u];
                if (t < L) a.dv[((size_t)(t0 + t) * H + h) * DV + c] = s_beta[t] * y[u];
            }
            st16(sm + BT_I7 + il_off(c, 16 * q4, 128), y);
            st16(sm + BT_I7 + il_off(c, 16 * q4 + 8, 128), y + 8);
            const float sum = lane_sum16(pr, lane);
            if ((lane & 1) == 0) atomicAdd(&s_db[16 * q4 + lane_sum16_token(lane)], sum);
        }
        images_ready();

        // ------------------------------------------------------------- stage 4
        if (tid == 0) {
            mma_run(tm + TB_S4A, desc_mn(sb + BT_I7, 128), step_mn(128), desc_mn(sb + BT_I12, 64), step_mn(64),
                    idesc_bf16_major(128, 64, 1, 1), 8, false);
            mma_run(tm + TB_S4B, desc_k(sb + BT_I5, 128), STEP_K, desc_mn(sb + BT_I7, 128), step_mn(128),
                    idesc_bf16_major(128, 128, 0, 1), 8, false);
            mma_commit(&bar[4]);
        }
        committed = 5;

        // ================================================================ phase E
        if (!wait_mma(4)) { failed = true; break; }
        {   // [-dM ; dP] rows -> [A' ; P'] image at their column versions, dbeta's dM o A part
            const int p = q4, r = 32 * qd + lane;
            const bool isP = r >= 64;
            const int t = r & 63, bt = t >> 4;
            float val[16], dmv[16];
            {
                float dd[16];
                tmem_ld16(lane_addr + TB_S4A + 16 * p, dd);
                tmem_ld_wait();
                const float bt_ = s_beta[t];
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) {
                    const int s = 16 * p + s16;
                    dmv[s16] = (!isP && s < t) ? -dd[s16] : 0.f;
                    val[s16] = isP ? ((s <= t) ? dd[s16] : 0.f) : bt_ * dmv[s16];
                }
            }
            if (!isP) {
                // dbeta += sum_s dM_ts A_ts over this piece: the unscaled A row piece from the
                // stage-1 accumulator, selected per lane from warp-uniform loads (tcgen05.ld
                // is warp-collective), as in the extraction
                float db2 = 0.f, aa[16];
                tmem_ld16(lane_addr + TB_AP + 16 * p, aa);
                tmem_ld_wait();
                if (p == bt) {
#pragma unroll
                    for (int s16 = 0; s16 < 16; ++s16) db2 += dmv[s16] * aa[s16];
                }
                if (qd == 0 && p == 0) {
                    tmem_ld16(lane_addr + TB_AP + SV_B1, aa);
                    tmem_ld_wait();
                    if (bt == 1) {
#pragma unroll
                        for (int s16 = 0; s16 < 16; ++s16) db2 += dmv[s16] * aa[s16];
                    }
                }
                if (qd == 1 && p < 2) {
                    tmem_ld16(lane_addr + TB_AP + SV_B2 + 16 * p, aa);
                    tmem_ld_wait();
                    if (bt == 2) {
#pragma unroll
                        for (int s16 = 0; s16 < 16; ++s16) db2 += dmv[s16] * aa[s16];
                    }
                }
                if (qd == 1 && p < 3) {
                    tmem_ld16(lane_addr + TB_AP + SV_B3 + 16 * p, aa);
                    tmem_ld_wait();
                    if (bt == 3) {
#pragma unroll
                        for (int s16 = 0; s16 < 16; ++s16) db2 += dmv[s16] * aa[s16];
                    }
                }
                if (p <= bt) atomicAdd(&s_db[t], db2);
            }
            uint8_t* row = sm + BT_I13;
            // Kd columns of tile p: the value on the diagonal block, zero elsewhere
            if (p == bt) {
                st16(row + il_off(r, 16 * p, NSV), val);
                st16(row + il_off(r, 16 * p + 8, NSV), val + 8);
            } else {
                st16z(row + il_off(r, 16 * p, NSV));
                st16z(row + il_off(r, 16 * p + 8, NSV));
            }
            // Kb pieces (6 of 16 columns): piece kb(bt) + p holds tile p < bt; the rest zero
            const int kb = bt == 1 ? 0 : bt == 2 ? 1 : 3;  // first value piece of this row's tile
            const int nval = bt;                           // value pieces: kb .. kb + bt - 1
            if (p < bt) {
                const uint32_t col = SV_B1 + 16u * (uint32_t)(kb + p);
                st16(row + il_off(r, col, NSV), val);
                st16(row + il_off(r, col + 8, NSV), val + 8);
            }
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const int piece = p + 4 * z;
                if (piece < 6 && !(bt > 0 && piece >= kb && piece < kb + nval)) {
                    const uint32_t col = SV_B1 + 16u * (uint32_t)piece;
                    st16z(row + il_off(r, col, NSV));
                    st16z(row + il_off(r, col + 8, NSV));
                }
            }
        }
        {   // KQr and KC again (their stage-1 copies were overwritten), now each as a high and a
            // low bf16 part: the row (KC) and column (KQr) forms of every A and P term must round
            // alike, or their contributions to dg, which cancel in dlog_alpha's chunk sums, stop
            // cancelling
            const float eD = __expf(Gs - Gn);
            const float f2 = __expf(((q4 == 0) ? G[2] : G[3]) - Gn);
            const float f3 = __expf(G[3] - Gn);
            float (&E1b)[16] = E1;
            float (&E3b)[16] = E3;
            if constexpr (IN_BF16) {  // from the log-decays kept since phase A
                float alpha[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int t = 16 * q4 + u;
                    const float raw = (u & 1) ? hi_bf(lar2[u >> 1]) : lo_bf(lar2[u >> 1]);
                    alpha[u] = __expf(t < L ? fmaxf(raw, -5.f) : 0.f);
                }
                E1b[0] = alpha[0];
#pragma unroll
                for (int u = 1; u < 16; ++u) E1b[u] = E1b[u - 1] * alpha[u];
                E3b[15] = 1.f;
#pragma unroll
                for (int u = 14; u >= 0; --u) E3b[u] = E3b[u + 1] * alpha[u + 1];
            } else {
                tile_decays<IN_BF16>(a, base_c, rowk, q4, L, E1b, E3b, &keep_la);
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int tf = 16 * q4 + 8 * m;
                float x[8], y[8], k3[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = 8 * m + e;
                    float kv, qv;
                    if (IN_BF16) {
                        kv = (u & 1) ? hi_bf(kr2[u >> 1]) : lo_bf(kr2[u >> 1]);
                        qv = (u & 1) ? hi_bf(qr2[u >> 1]) : lo_bf(qr2[u >> 1]);
                    } else {
                        const int t = tf + e;
                        kv = t < L ? ld_in(a.k, base_c + (size_t)t * rowk, 0) : 0.f;
                        qv = t < L ? ld_in(a.q, base_c + (size_t)t * rowk, 0) : 0.f;
                    }
                    x[e] = kv * E1b[u];
                    y[e] = qv * E1b[u] * a.scale;
                    k3[e] = kv * E3b[u];
                }
                st16_hilo(sm + BT_I1B + il_off(c, tf, 128), sm + BT_I1L + il_off(c, tf, 128), x);
                st16_hilo(sm + BT_I1B + il_off(c, 64 + tf, 128), sm + BT_I1L + il_off(c, 64 + tf, 128), y);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = k3[e] * eD;
                st16_hilo(sm + BT_I2B + il_off(c, tf, NSV), sm + BT_I2L + il_off(c, tf, NSV), x);
                if (q4 == 0) {
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B1 + tf, NSV), sm + BT_I2L + il_off(c, SV_B1 + tf, NSV), k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f2;
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B2 + tf, NSV), sm + BT_I2L + il_off(c, SV_B2 + tf, NSV), x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f3;
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B3 + tf, NSV), sm + BT_I2L + il_off(c, SV_B3 + tf, NSV), x);
                } else if (q4 == 1) {
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B2 + tf, NSV), sm + BT_I2L + il_off(c, SV_B2 + tf, NSV), k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = k3[e] * f3;
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B3 + tf, NSV), sm + BT_I2L + il_off(c, SV_B3 + tf, NSV), x);
                } else if (q4 == 2) {
                    st16_hilo(sm + BT_I2B + il_off(c, SV_B3 + tf, NSV), sm + BT_I2L + il_off(c, SV_B3 + tf, NSV), k3);
                }
            }
        }
        images_ready();

        // ------------------------------------------------------------- stage 5
        if (tid == 0) {
            mma_run(tm + TB_S5A, desc_k(sb + BT_I2B, NSV), STEP_K, desc_k(sb + BT_I13, NSV), STEP_K,
                    idesc_bf16_major(128, 128, 0, 0), NSV / 16, false);
            mma_run(tm + TB_S5A, desc_k(sb + BT_I2L, NSV), STEP_K, desc_k(sb + BT_I13, NSV), STEP_K,
                    idesc_bf16_major(128, 128, 0, 0), NSV / 16, true);
            mma_run(tm + TB_S5B, desc_k(sb + BT_I1B, 128), STEP_K, desc_mn(sb + BT_I13, NSV), step_mn(NSV),
                    idesc_bf16_major(128, 160, 0, 1), 8, false);
            mma_run(tm + TB_S5B, desc_k(sb + BT_I1L, 128), STEP_K, desc_mn(sb + BT_I13, NSV), step_mn(NSV),
                    idesc_bf16_major(128, 160, 0, 1), 8, true);
            mma_commit(&bar[5]);
        }
        committed = 6;

        // ================================================================ phase F
        if (!wait_mma(5)) { failed = true; break; }
        {
            const float eG = __expf(Gs), eC = __expf(G[4] - Gn), eD = __expf(Gs - Gn);
            const float f2 = __expf(((q4 == 0) ? G[2] : G[3]) - Gn);
            const float f3 = __expf(G[3] - Gn);
            float* s_dg = reinterpret_cast<float*>(sm);  // [64 t][128 c]: every image is dead now
            float dgc = 0.f, tot = 0.f;
#pragma unroll 1
            for (int m = 0; m < 2; ++m) {
                const uint32_t cu = 16u * q4 + 8u * m;
                // this half's raw k, scale * q and decay factors (selected, not indexed, so that
                // they stay in registers)
                auto kv = [&](int e) -> float {
                    const int u = 8 * m + e, t = 16 * q4 + u;
                    if (IN_BF16) {
                        const uint32_t w = m ? kr2[4 + (e >> 1)] : kr2[e >> 1];
                        return (e & 1) ? hi_bf(w) : lo_bf(w);
                    }
                    return t < L ? ld_in(a.k, base_c + (size_t)t * rowk, 0) : 0.f;
                };
                auto qb = [&](int e) -> float {
                    const int u = 8 * m + e, t = 16 * q4 + u;
                    if (IN_BF16) {
                        const uint32_t w = m ? qr2[4 + (e >> 1)] : qr2[e >> 1];
                        return a.scale * ((e & 1) ? hi_bf(w) : lo_bf(w));
                    }
                    return t < L ? a.scale * ld_in(a.q, base_c + (size_t)t * rowk, 0) : 0.f;
                };
                auto e1 = [&](int e) -> float { return m ? E1[8 + e] : E1[e]; };
                auto e3 = [&](int e) -> float { return m ? E3[8 + e] : E3[e]; };
                float dq8[8], dk8[8], dg8[8], x[8];
                // q: through the state, dO S0^T scaled by Gam; through P's rows
                tmem_ld8(lane_addr + TB_S4B + 64 + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = e1(e) * eG * x[e];
                    dq8[e] = w;
                    dg8[e] = qb(e) * w;
                }
                tmem_ld8(lane_addr + TB_S5A + 64 + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = e1(e) * x[e];
                    dq8[e] += w;
                    dg8[e] += qb(e) * w;
                    const int t = (int)cu + e;
                    if (t < L) a.dq[base_c + (size_t)t * rowk] = a.scale * dq8[e];
                }
                // k: through R, -(beta Y) S0^T scaled by Gam
                tmem_ld8(lane_addr + TB_S4B + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = -s_beta[cu + e] * x[e] * e1(e) * eG;
                    dk8[e] = w;
                    dg8[e] += kv(e) * w;
                }
                // k: through the chunk-end state, U dS_C^T scaled by e^{g_C - g}
                tmem_ld8(lane_addr + TB_KC + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = x[e] * e3(e) * eC;
                    dk8[e] += w;
                    dg8[e] -= kv(e) * w;
                    dgc += kv(e) * w;
                }
                // k: A's rows (t as the row token)
                tmem_ld8(lane_addr + TB_S5A + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = e1(e) * x[e];
                    dk8[e] += w;
                    dg8[e] += kv(e) * w;
                }
                // k: A's and P's columns (t as the column token): its versions, each with its factor
                tmem_ld8(lane_addr + TB_S5B + cu, x);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float w = e3(e) * eD * x[e];
                    dk8[e] += w;
                    dg8[e] -= kv(e) * w;
                }
                if (q4 <= 2) {  // the version of tile q4 + 1: factor e^{G_{q4+1} - g} = E3
                    const uint32_t base = q4 == 0 ? SV_B1 : q4 == 1 ? SV_B2 + 16 : SV_B3 + 32;
                    tmem_ld8(lane_addr + TB_S5B + base + 8u * m, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float w = e3(e) * x[e];
                        dk8[e] += w;
                        dg8[e] -= kv(e) * w;
                    }
                }
                if (q4 <= 1) {  // tile q4 + 2
                    const uint32_t base = q4 == 0 ? SV_B2 : SV_B3 + 16;
                    tmem_ld8(lane_addr + TB_S5B + base + 8u * m, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float w = e3(e) * f2 * x[e];
                        dk8[e] += w;
                        dg8[e] -= kv(e) * w;
                    }
                }
                if (q4 == 0) {  // tile 3
                    tmem_ld8(lane_addr + TB_S5B + SV_B3 + 8u * m, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float w = e3(e) * f3 * x[e];
                        dk8[e] += w;
                        dg8[e] -= kv(e) * w;
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = (int)cu + e;
                    tot += dg8[e];
                    s_dg[t * 128 + c] = dg8[e];
                    if (t < L) a.dk[base_c + (size_t)t * rowk] = dk8[e];
                }
            }
            // dlog_alpha: reverse cumulative sum of dg over the chunk plus dL/dg_C
            s_tot[q4 * 128 + c] = tot;
            s_dgc[q4 * 128 + c] = dgc;
            __syncthreads();
            float run = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                run += s_dgc[qq * 128 + c] + __expf(G[4]) * s_rs[qq * 128 + c];
                if (qq > q4) run += s_tot[qq * 128 + c];
            }
#pragma unroll
            for (int u = 15; u >= 0; --u) {
                const int t = 16 * q4 + u;
                run += s_dg[t * 128 + c];
                if (t < L) a.dla[base_c + (size_t)t * rowk] = (keep_la >> u) & 1u ? run : 0.f;
            }
            if (tid < CH && tid < L) a.dbeta[(size_t)(t0 + tid) * H + h] = s_db[tid];
        }
        tc_fence_before();
        __syncthreads();  // shared memory and TMEM are reused by the next item
        tc_fence_after();
        par ^= 1u;
        committed = 0;
    }
    if (failed && tid == 0) {
        // tile loads and products still in flight complete before the CTA retires (bounded)
        if (committed == 7) mbar_wait(&bar[6], par, nullptr);
        else if (committed == 8) mbar_wait(&bar[7], par, nullptr);
        else
            for (int i = 0; i < committed; ++i) mbar_wait(&bar[i], par, nullptr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ------------------------------------------------ reverse chain (tensor cores)
// One CTA per (sequence, head, 32-column slice js of dS), warp-specialised like the
// forward chain: warps 0-3 own one row i of the dS slice each (32 fp32 registers),
// warp 4 (one thread) issues the tensor-core products, warp 5 (one thread) bulk-loads
// each chunk's M_lr, Q' and Gamma_C from the forward's workspace slot, three chunks ahead.
// Per chunk c, in reverse:
//     dS_end[c] = dS;   dS <- Gamma_C o dS + D,   D = Q'^T dO_c - M_lr^T dS
// D (M = 128 rows i, N = 32 columns) accumulates in TMEM: Q'^T dO_c first (it does not
// depend on dS, so it is issued one chunk ahead, off the sequential path), then M_lr^T
// (-dS) on top.  M_lr^T is the slot's K-major 128-byte-swizzle M_lr image read as an
// MN-major operand; Q'^T is the slot's token-contiguous Q' image read as a K-major one.
// dO_c enters as a bf16 image [32 j][64 t] written by the consumers from registers
// loaded one chunk ahead; -dS as a bf16 image [128 m][32 j].
constexpr int RB_THREADS = 192;
constexpr int RB_NBUF = 3;
constexpr uint32_t RB_SLOT = 50176;                    // M_lr + Q' + Gamma_C (49,664 B), 1024-aligned stride
constexpr uint32_t RB_DS = RB_NBUF * RB_SLOT;          // -dS image [128 m][32 j] bf16
constexpr uint32_t RB_DO = RB_DS + 8192;               // dO images [2][32 j][64 t] bf16
constexpr uint32_t RB_BAR = RB_DO + 8192;
constexpr uint32_t RB_TPTR = RB_BAR + 128;
constexpr uint32_t RB_SMEM = RB_TPTR + 16 + 1024;
static_assert(RB_SLOT >= SO_MQG && RB_SLOT % 1024 == 0, "slot buffer stride");

// M_lr^T from the K-major 128-byte-swizzle M_lr image: MN-major operand, 64-element MN
// blocks 16,384 B apart, 8-row K groups 1,024 B apart
KDA_DEV uint64_t sdesc_mn_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16384u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
// element (t, j) of a dO image: 8-column blocks 1,024 B apart, token rows 16 B apart
KDA_DEV uint32_t do_off(uint32_t t, uint32_t j) { return (j >> 3) * 1024u + t * 16u + (j & 7u) * 2u; }

template <bool IN_BF16>
__global__ void __launch_bounds__(RB_THREADS, 1) chain_bwd_tc_kernel(const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int js = blockIdx.x, h = blockIdx.y, n = blockIdx.z, H = a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool consumer = warp < 4;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + RB_BAR);          // [3]
    uint64_t* bar_free = reinterpret_cast<uint64_t*>(sm + RB_BAR + 24);   // [3]
    uint64_t* bar_img = reinterpret_cast<uint64_t*>(sm + RB_BAR + 48);
    uint64_t* bar_d = reinterpret_cast<uint64_t*>(sm + RB_BAR + 56);      // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + RB_TPTR);
    int64_t s_beg, s_end;
    bwd_seq_range(a, n, s_beg, s_end);
    const int nck = (int)((s_end - s_beg + CH - 1) / CH);
    // this consumer's row i = tid, columns [32 js, 32 js + 32)
    const size_t st = ((size_t)n * H + h) * STATE + (size_t)(consumer ? tid : 0) * DV + (size_t)DVS * js;
    float dS[DVS];
    if (consumer) {
#pragma unroll
        for (int j = 0; j < DVS; j += 4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.d_final) v4 = *reinterpret_cast<const float4*>(a.d_final + st + j);
            dS[j] = v4.x; dS[j + 1] = v4.y; dS[j + 2] = v4.z; dS[j + 3] = v4.w;
        }
    }
    if (nck > 0) {
        if (warp == 0) {
            tmem_alloc(s_tmem, 64);
            tmem_relinquish();
        }
        if (tid == 0) {
            for (int i = 0; i < RB_NBUF; ++i) {
                mbar_init(&bar_ld[i], 1);
                mbar_init(&bar_free[i], 128);
            }
            mbar_init(bar_img, 128);
            mbar_init(&bar_d[0], 1);
            mbar_init(&bar_d[1], 1);
            fence_mbar_init();
        }
        __syncthreads();
        tc_fence_after();
        const uint32_t tm = *s_tmem;
        // iteration it handles chunk c = nck - 1 - it
        auto slot_of = [&](int it) {
            return a.slots + (((size_t)n * a.wc + (nck - 1 - it)) * H + h) * SLOT_BYTES;
        };
        auto bidx = [](int it) { return it % RB_NBUF; };
        auto bpar = [](int it) { return (uint32_t)((it / RB_NBUF) & 1); };
        bool failed = false;
        int loads_issued = 0, mma_issued = 0;

        if (warp == 5) {
            // ------------------------------------------------------------ loader
            if (lane == 0) {
                auto issue_load = [&](int it) {
                    const int b = bidx(it);
                    mbar_arrive_expect_tx(&bar_ld[b], SO_MQG);
                    bulk_g2s(sm + b * RB_SLOT, slot_of(it) + SO_M, SO_MQG, &bar_ld[b]);
                };
                for (int j = 0; j < RB_NBUF && j < nck; ++j) {
                    issue_load(j);
                    loads_issued = j + 1;
                }
                for (int j = 0; j + RB_NBUF < nck; ++j) {
                    if (!mbar_wait(&bar_free[bidx(j)], bpar(j), a.status)) {
                        failed = true;
                        break;
                    }
                    issue_load(j + RB_NBUF);
                    loads_issued = j + RB_NBUF + 1;
                }
            }
        } else if (warp == 4) {
            // ------------------------------------------------------ tensor issue
            if (lane == 0) {
                const uint32_t id1 = idesc_bf16_major(128, DVS, 1, 1), id2 = idesc_bf16_major(128, DVS, 0, 1);
                // Q'^T dO of iteration it into accumulator it & 1 (overwrites)
                auto issue_qdo = [&](int it) {
                    const uint32_t buf = sbase + bidx(it) * RB_SLOT;
                    const uint64_t ad = sdesc_interleave(buf + SO_Q, 128u, 1024u);
                    const uint64_t bd = sdesc_interleave(sbase + RB_DO + (it & 1) * 4096, 128u, 1024u);
#pragma unroll
                    for (int kk = 0; kk < CH / 16; ++kk)
                        mma_bf16(tm + 32 * (it & 1), ad + (uint32_t)((kk * 256) >> 4), bd + (uint32_t)((kk * 256) >> 4), id2,
                                 kk > 0 ? 1u : 0u);
                };
                // the first chunk's dO image (announced on bar_img's phase 0) and slot
                if (!mbar_wait(bar_img, 0u, a.status) || !mbar_wait(&bar_ld[bidx(0)], bpar(0), a.status)) {
                    failed = true;
                } else {
                    tc_fence_after();
                    issue_qdo(0);
                    for (int it = 0; it < nck; ++it) {
                        // the -dS image of this chunk (and the dO image of the next one)
                        if (!mbar_wait(bar_img, (uint32_t)((it + 1) & 1), a.status)) {
                            failed = true;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t md = sdesc_mn_sw128(sbase + bidx(it) * RB_SLOT + SO_M);
                        const uint64_t sd = sdesc_interleave(sbase + RB_DS, 512u, 128u);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            mma_bf16(tm + 32 * (it & 1), md + (uint32_t)((kk * 2048) >> 4),
                                     sd + (uint32_t)((kk * 1024) >> 4), id1, 1u);
                        mma_commit(&bar_d[it & 1]);
                        mma_issued = it + 1;
                        if (it + 1 < nck) {
                            if (!mbar_wait(&bar_ld[bidx(it + 1)], bpar(it + 1), a.status)) {
                                failed = true;
                                break;
                            }
                            tc_fence_after();
                            issue_qdo(it + 1);
                        }
                    }
                }
            }
        } else {
            // --------------------------------------------------------- consumers
            const int i = tid;
            const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
            // dO of iteration it: token t = i / 2, 16 columns from 16 (i % 2), bf16 bits in registers
            uint32_t dw[8];
            auto load_do = [&](int it) {
#pragma unroll
                for (int e = 0; e < 8; ++e) dw[e] = 0u;
                if (it >= nck) return;
                const int c = nck - 1 - it;
                const int t = i >> 1;
                const int64_t tok = s_beg + (int64_t)c * CH + t;
                if (tok >= s_end) return;
                const size_t base = ((size_t)tok * H + h) * DV + (size_t)DVS * js + 16 * (i & 1);
                if constexpr (IN_BF16) {
                    const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.d_o) + base));
                    const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.d_o) + base + 8));
                    dw[0] = u0.x; dw[1] = u0.y; dw[2] = u0.z; dw[3] = u0.w;
                    dw[4] = u1.x; dw[5] = u1.y; dw[6] = u1.z; dw[7] = u1.w;
                } else {
                    const float* src = reinterpret_cast<const float*>(a.d_o) + base;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 f = __ldg(reinterpret_cast<const float4*>(src) + e);
                        dw[2 * e] = pack_bf16x2(f.x, f.y);
                        dw[2 * e + 1] = pack_bf16x2(f.z, f.w);
                    }
                }
            };
            auto write_do = [&](int it) {
                uint8_t* img = sm + RB_DO + (it & 1) * 4096;
                const int t = i >> 1, jb = 2 * (i & 1);
                *reinterpret_cast<uint4*>(img + do_off((uint32_t)t, 8u * jb)) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
                *reinterpret_cast<uint4*>(img + do_off((uint32_t)t, 8u * (jb + 1))) = make_uint4(dw[4], dw[5], dw[6], dw[7]);
            };
            load_do(0);
            write_do(0);
            load_do(1);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bar_img);
            for (int it = 0; it < nck; ++it) {
                const int c = nck - 1 - it, b = bidx(it);
                // dL/d(state at the end of chunk c), as a bf16 operand image (row i, this slice's columns)
                uint8_t* dimg = a.ds_end + (((size_t)n * a.wc + c) * H + h) * STATE_IMG_BYTES;
#pragma unroll
                for (int m = 0; m < DVS / 8; ++m)
                    *reinterpret_cast<uint4*>(dimg + state_img_off((uint32_t)i, (uint32_t)(DVS * js + 8 * m))) =
                        pack8f(dS + 8 * m);
                // -dS image (row m = i) and the next chunk's dO image
                {
                    uint8_t* img = sm + RB_DS + (uint32_t)(i >> 3) * 512u + (uint32_t)(i & 7) * 16u;
                    float ng[8];
#pragma unroll
                    for (int jb = 0; jb < DVS / 8; ++jb) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) ng[e] = -dS[8 * jb + e];
                        *reinterpret_cast<uint4*>(img + jb * 128) = pack8f(ng);
                    }
                }
                if (it + 1 < nck) {
                    write_do(it + 1);
                    load_do(it + 2);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bar_img);
                if (!mbar_wait(&bar_d[it & 1], (uint32_t)((it >> 1) & 1), a.status) ||
                    !mbar_wait(&bar_ld[b], bpar(it), a.status)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float d[DVS];
                tmem_ld32(lane_addr + 32 * (it & 1), d);
                tmem_ld_wait();
                const float gam = *reinterpret_cast<const float*>(sm + b * RB_SLOT + SO_G + 4 * i);
#pragma unroll
                for (int j = 0; j < DVS; ++j) dS[j] = gam * dS[j] + d[j];
                tc_fence_before();
                mbar_arrive(&bar_free[b]);
            }
        }
        // copies and products in flight finish before the CTA retires (bounded)
        __syncthreads();
        if (warp == 5 && lane == 0) {
            for (int j = loads_issued - RB_NBUF < 0 ? 0 : loads_issued - RB_NBUF; j < loads_issued; ++j)
                mbar_wait(&bar_ld[bidx(j)], bpar(j), nullptr);
        }
        if (warp == 4 && lane == 0 && failed && mma_issued > 0) {
            const int j = mma_issued - 1;
            mbar_wait(&bar_d[j & 1], (uint32_t)((j >> 1) & 1), nullptr);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tm, 64);
        if (failed) return;
    }
    if (consumer && a.d_init) {
#pragma unroll
        for (int j = 0; j < DVS; j += 4)
            *reinterpret_cast<float4*>(a.d_init + st + j) = make_float4(dS[j], dS[j + 1], dS[j + 2], dS[j + 3]);
    }
}

}  // namespace

size_t chunk_bwd_extra_bytes(int n_seqs, int H, int64_t max_seqlen) {
    const int64_t nck = (max_seqlen + CH - 1) / CH;
    const int64_t n_ckpt = max_seqlen / CH;
    return (size_t)n_seqs * H * STATE_IMG_BYTES * (size_t)(nck + n_ckpt);
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
        if ((err = cudaFuncSetAttribute(chain_bwd_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)RB_SMEM)) != cudaSuccess ||
            (err = cudaFuncSetAttribute(chain_bwd_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)RB_SMEM)) != cudaSuccess ||
            (err = cudaFuncSetAttribute(bwd_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)BT_SMEM)) != cudaSuccess ||
            (err = cudaFuncSetAttribute(bwd_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)BT_SMEM)) != cudaSuccess)
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
    uint8_t* ckpt = ws + fwd_bytes;  // chunk-boundary states, bf16 images
    uint8_t* ds_end = ckpt + (size_t)N * n_ckpt * H * STATE_IMG_BYTES;
    // 1. the forward walk again, without outputs: chunk slots and chunk-boundary states
    err = chunk_fwd_launch(q, k, v, log_alpha, beta, init_state, nullptr, nullptr, B, T, H, cu, n_seqs, max_seqlen,
                           in_bf16, false, scale, nullptr, nullptr, 0.f, n_ckpt > 0 ? reinterpret_cast<float*>(ckpt) : nullptr, CH, 1, KCP_NONE,
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
    if (in_bf16) chain_bwd_tc_kernel<true><<<dim3(NSL, H, N), RB_THREADS, RB_SMEM, stream>>>(a);
    else chain_bwd_tc_kernel<false><<<dim3(NSL, H, N), RB_THREADS, RB_SMEM, stream>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    prof_end(PROF_CHAIN_BWD, stream);
    // 3. the chunk-local gradients
    const int64_t n_items = (int64_t)N * a.wc * H;
    if (nck > 0 && n_items > 0) {
        const unsigned grid = (unsigned)(n_items < sms ? n_items : sms);
        BwdMaps maps;
        memset(&maps, 0, sizeof(maps));
        const int64_t total_tokens = cu ? T : (int64_t)B * T;
        if (in_bf16 && (!make_bf16_tile_map(&maps.la, log_alpha, total_tokens, (int64_t)H * DK) ||
                        !make_bf16_tile_map(&maps.k, k, total_tokens, (int64_t)H * DK) ||
                        !make_bf16_tile_map(&maps.q, q, total_tokens, (int64_t)H * DK) ||
                        !make_bf16_tile_map(&maps.v, v, total_tokens, (int64_t)H * DV) ||
                        !make_bf16_tile_map(&maps.d_o, d_o, total_tokens, (int64_t)H * DV)))
            return cudaErrorInvalidValue;
        prof_begin(PROF_INTRA_BWD, stream);
        if (in_bf16) bwd_tc_kernel<true><<<grid, BT_THREADS, BT_SMEM, stream>>>(a, maps, n_items);
        else bwd_tc_kernel<false><<<grid, BT_THREADS, BT_SMEM, stream>>>(a, maps, n_items);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        prof_end(PROF_INTRA_BWD, stream);
    }
    return cudaSuccess;
}

}  // namespace kda
