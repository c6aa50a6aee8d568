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
//   intra_kernel  persistent, one CTA per SM, loops over (chunk, head) items.
//                 Raw q/k/v/log_alpha tiles arrive by TMA (2-D tensor maps),
//                 prefetched one item ahead.  Builds the decay-scaled operands,
//                 runs every product above on the tensor cores (tcgen05.mma,
//                 fp32 accumulators in TMEM), inverts the 64x64 unit-triangular
//                 system in fp32, and writes Mlr, Qp, Gam_C, Bm, Ob to one
//                 workspace slot per (chunk, head).
//   chain_kernel  one CTA per (value-column slice, head, sequence); walks the
//                 chunks in order.  Per chunk ONE tensor-core product on the
//                 sequential path (Mlr S, the state slice as the B operand),
//                 then S <- Gam_C o S - Mlr S + Bm in fp32 registers; the
//                 output product Qp S (+ Ob) runs beside it off the critical
//                 path.  Every per-chunk operand arrives by bulk copies (TMA
//                 engine), two chunks ahead.
//
// Exponent references (why the -5 bound matters): inside a 64-token chunk the
// cumulative decay can reach e^{-320}, whose reciprocal overflows fp32/bf16.
// Each 16-token tile b uses its own reference G_b = g at the token before the
// tile (G_0 = 0).  Row operands carry e^{g_t - G_b} <= 1; column operands of
// the diagonal tile carry e^{G_b - g_s} <= e^{16*5} = e^80 (finite in bf16);
// column operands of earlier tiles carry e^{G_b - g_s} = e^{G_b - G_{bs+1}}
// e^{G_{bs+1} - g_s}, a product of two factors <= 1.  Every bf16 operand is
// finite and every product is a correctly-scaled e^{g_t - g_s}.
#include <cudaTypedefs.h>
#include <string.h>

#include "kda_launch.h"
#include "kda_profile.h"
#include "kda_sm100.cuh"
#include "kda_slots.h"
#include "kda_tri.cuh"

namespace kda {

// chunk length, head dims and the workspace slot layout: kda_slots.h

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
    uint8_t* ws;               // slots
    uint32_t* status;
    int64_t T;                 // tokens per sequence (fixed) or total tokens (varlen)
    int H;
    int n_seqs;
    int i0;                    // first chunk index of this pass (within each sequence)
    int wc;                    // chunk slots per sequence in this pass
    int first_pass;
    float scale;
    float* ckpt;               // nullable: states at every ckpt_every-th chunk boundary
    int ckpt_every;            // in chunks
    int n_ckpt;                // checkpoints per sequence in `ckpt`
    int segs;                  // segments per sequence (segment-parallel prefill), else 1
    uint8_t* seg_ws;           // segment transition slots [n_seqs][segs][H], segment-parallel only
    float* trans_out;          // nullable: fp32 segment maps [2][n_seqs][H][dk][dk] (M, then B) instead of slots
    unsigned long long wait_ns;  // limit of the intra kernel's tile-load wait (WAIT_LIMIT_NS unless a test shortens it)
    int drop_tile;             // test hook: CTA 0 does not issue one tile load of its first item (its wait runs out)
    int wait_first;            // the kernel ahead of the chain may be the caller's (the cross-device finish,
                               // whose initial state the fold wrote): the chain waits for it before reading
                               // anything, not only before the slots
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

// Item = workspace slot = ((n * wc) + (chunk - i0)) * H + h.  Returns false if
// that chunk lies beyond its sequence.
KDA_DEV bool item_info(const ChunkArgs& a, int64_t item, int& h, int64_t& t0, int& L) {
    const uint32_t it32 = (uint32_t)item;  // items per pass < 2^31
    const uint32_t rest = it32 / (uint32_t)a.H;
    h = (int)(it32 - rest * (uint32_t)a.H);
    const uint32_t nn = rest / (uint32_t)a.wc;
    const int n = (int)nn;
    const int ci = a.i0 + (int)(rest - nn * (uint32_t)a.wc);
    int64_t sb, se;
    seq_range(a, n, sb, se);
    t0 = sb + (int64_t)ci * CH;
    if (t0 >= se) return false;
    L = (int)((se - t0) < CH ? (se - t0) : CH);
    return true;
}

// Issues D (+)= A B^T over K = 16 * NK for two K-major SW128 images given by
// their base descriptors.  A_ROWS / B_ROWS are the row counts of one
// 128-byte-wide K block of each.  A descriptor's start-address field is the
// byte address / 16 in its low bits, so stepping K adds (byte offset / 16).
template <int NK, int A_ROWS, int B_ROWS>
KDA_DEV void mma_sw128(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
        const uint32_t ao = ((uint32_t)(kk >> 2) * A_ROWS * 128u + (uint32_t)(kk & 3) * 32u) >> 4;
        const uint32_t bo = ((uint32_t)(kk >> 2) * B_ROWS * 128u + (uint32_t)(kk & 3) * 32u) >> 4;
        mma_bf16(d, adesc + ao, bdesc + bo, idesc, kk > 0 ? 1u : 0u);
    }
}

// Same for two MN-major no-swizzle images (core-matrix M/N stride 128 B; K-group
// stride A_KG / B_KG bytes): one MMA step of K = 16 spans two K groups.
template <int NK, int A_KG, int B_KG>
KDA_DEV void mma_mn(uint32_t d, uint32_t a_addr, uint32_t b_addr, uint32_t idesc) {
    const uint64_t ad0 = sdesc_interleave(a_addr, A_KG, 128u), bd0 = sdesc_interleave(b_addr, B_KG, 128u);
#pragma unroll
    for (int kk = 0; kk < NK; ++kk)
        mma_bf16(d, ad0 + (uint32_t)((kk * 2 * A_KG) >> 4), bd0 + (uint32_t)((kk * 2 * B_KG) >> 4), idesc,
                 kk > 0 ? 1u : 0u);
}

// Position of 16-byte piece m of row r in a 64-byte-row slice (see the slot layout).
KDA_DEV uint32_t swz64(uint32_t r, uint32_t m) { return m ^ ((r >> 1) & 3u); }

KDA_DEV uint4 pack8(const float* x) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
}

// ---------------------------------------------------------------------------
// intra_kernel
// ---------------------------------------------------------------------------
// Threads: 512.  Thread tid owns key/value channel c = tid & 127 and the
// 16-token tile q4 = tid >> 7 (tokens [16 q4, 16 q4 + 16)).  Warp w reads TMEM
// lanes 32*(w & 3) .. +31 (rows c = tid & 127); its group w >> 2 = q4 picks
// the columns it extracts.
//
// Shared memory (offsets from a 1024-aligned base):
//   RAW [0, 64K)     TMA tiles [64 tokens][128 ch] bf16: la @0, k @16K, q @32K, v @48K
//   X   [64K, 136K)  phase 1 (MN-major, no swizzle, M/N = token): KQr 128x128 @0,
//                             KC = [Kd 64 | Kb1 16 | Kb2 32 | Kb3 48] x 128 @32K
//                    after stage 1: Ti [64][64] @32K, Ph [64][64] @56K, inverse scratch @64K
//   Y   [136K, 171K) A fp32 [64][68] @0, X fp32 [64][68] @17408;
//                    later Wt [128][64] @0, Ut [128][64] @16K
//   Z2  [171K, 219K) KGt, Vt, Ktt [128][64] (built while stage 1 runs)
//   misc             beta[64], G[5][128], tile totals[4][128], 2 mbarriers, TMEM base
// The workspace slot is assembled in two regions ([Mlr | Qp | GamC] at X, [Bm | Ob]
// at Z2) and leaves as four bulk copies: Mlr and Bm as soon as they are staged, the
// rest at the end of the item.
// TMEM (512 columns): stage 1  A/P diag [0,64), off-diag [64,80) [80,112) [112,160)
//                     stage 2  Wt [160,224), Ut [224,288)
//                     stage 3  [Mlr | Bm] [0,256) (one N = 256 product), (PW)^T [256,320),
//                              Ob = P Ut^T [320,448) (M = 64: token t in lane 32 (t / 16) + t % 16)
constexpr int INTRA_THREADS = 512;
constexpr uint32_t R_LA = 0, R_K = 16384, R_Q = 32768, R_V = 49152;
constexpr uint32_t IX = 65536;
// KC stacks the column operands of stage 1 as N = 160 token rows of one MN-major image:
// rows [0,64) Kd, [64,80) Kb1, [80,112) Kb2, [112,160) Kb3 (K-group stride 160 * 16 B).
constexpr uint32_t IX_KQR = IX + 0, IX_KC = IX + 32768;
constexpr uint32_t KC_KG = 2560, KC_B1 = 64, KC_B2 = 80, KC_B3 = 112;
constexpr uint32_t IX_TI = IX + 32768, IX_PH = IX + 57344, IX_TMP = IX + 65536;
constexpr uint32_t IY = IX + 73728;
constexpr int LDA = 68;  // padded fp32 row stride of A and X (16-byte rows, spread banks)
constexpr uint32_t IY_A = IY, IY_X = IY + 64 * LDA * 4, IY_WT = IY, IY_UT = IY + 16384;
// Z2: the phase-2 operand images (built while stage 1 runs), K-major SW128 [128 ch][64 tok]
constexpr uint32_t Z2 = IY + 35840;
constexpr uint32_t Z2_KGT = Z2, Z2_VT = Z2 + 16384, Z2_KTT = Z2 + 32768;
constexpr uint32_t IM = Z2 + 49152;
constexpr uint32_t IM_BETA = IM, IM_G = IM + 256, IM_TOT = IM + 256 + 2560, IM_BAR_RAW = IM_TOT + 2048,
                   IM_BAR_MMA = IM_BAR_RAW + 8, IM_BAR_MMA2 = IM_BAR_MMA + 8, IM_NEXT = IM_BAR_MMA2 + 8,
                   IM_TMEM = IM_NEXT + 32;
constexpr uint32_t INTRA_SMEM = IM_TMEM + 16 + 1024;  // + alignment slack
constexpr uint32_t INTRA_TMEM_COLS = 512;
constexpr uint32_t TM_AD = 0, TM_B1 = 64, TM_B2 = 80, TM_B3 = 112, TM_WT = 160, TM_UT = 224, TM_M = 0,
                   TM_BM = 128, TM_PW = 256, TM_OB = 320;

struct IntraMaps {
    CUtensorMap la, k, q, v;
};

// Raw bf16 bits of (token t, channel c) of a TMA tile, 0 past the chunk's end.
KDA_DEV uint32_t raw_bits(const uint8_t* sm, uint32_t tile, int t, int c, int L) {
    return (t < L) ? (uint32_t)*reinterpret_cast<const uint16_t*>(sm + tile + (uint32_t)(t * 128 + c) * 2u) : 0u;
}

template <bool IN_BF16>
KDA_DEV float raw_in(const uint8_t* sm, uint32_t tile, const void* gsrc, size_t ebase, size_t rowstride, int t,
                     int c, int L) {
    if (t >= L) return 0.f;
    if constexpr (IN_BF16) {
        return bf16_to_f32(*reinterpret_cast<const uint16_t*>(sm + tile + (uint32_t)(t * 128 + c) * 2u));
    } else {
        return __ldg(reinterpret_cast<const float*>(gsrc) + ebase + (size_t)t * rowstride);
    }
}

template <bool IN_BF16>
__global__ void __launch_bounds__(INTRA_THREADS, 1)
intra_kernel(const ChunkArgs a, const __grid_constant__ IntraMaps maps, const int64_t n_items) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = tid & 127, q4 = tid >> 7;
    const int qd = warp & 3;
    const int H = a.H;

    float* s_beta = reinterpret_cast<float*>(sm + IM_BETA);
    float* s_G = reinterpret_cast<float*>(sm + IM_G);      // [5][128]
    float* s_tot = reinterpret_cast<float*>(sm + IM_TOT);  // [4][128]
    uint64_t* bar_raw = reinterpret_cast<uint64_t*>(sm + IM_BAR_RAW);
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + IM_BAR_MMA);
    uint64_t* bar_mma2 = reinterpret_cast<uint64_t*>(sm + IM_BAR_MMA2);  // second half of stage 3
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + IM_TMEM);
    // next item of this CTA: {item, t0} as int64 and {h, L} as int
    int64_t* s_next64 = reinterpret_cast<int64_t*>(sm + IM_NEXT);
    int* s_next32 = reinterpret_cast<int*>(sm + IM_NEXT + 16);

    if (warp == 0) {
        tmem_alloc(s_tmem, INTRA_TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_mma2, 1);
        fence_mbar_init();
        if constexpr (IN_BF16) {
            prefetch_tmap(&maps.la);
            prefetch_tmap(&maps.k);
            prefetch_tmap(&maps.q);
            prefetch_tmap(&maps.v);
        }
    }
    __syncthreads();
    tc_fence_after();
    // the chain launch that follows may be scheduled now: its CTAs take SMs as this
    // kernel's CTAs retire and wait (pdl_wait) for the whole of this kernel
    pdl_trigger();
    const uint32_t tm = *s_tmem;
    const uint32_t lane_addr = tm + ((uint32_t)(32 * qd) << 16);
    uint32_t ph_raw = 0, ph_mma = 0, ph_mma2 = 0;

    // next valid item at or after `from` (stride gridDim.x), or n_items
    auto next_valid = [&](int64_t from) -> int64_t {
        for (int64_t it = from; it < n_items; it += gridDim.x) {
            int hh, LL;
            int64_t tt;
            if (item_info(a, it, hh, tt, LL)) return it;
        }
        return n_items;
    };
    // drop: the test hook's missing tile (the barrier still expects its bytes)
    auto issue_raw = [&](int hh, int64_t tt, bool drop) {
        mbar_arrive_expect_tx(bar_raw, 4u * 16384u);
        tma_load_2d(sm + R_LA, &maps.la, hh * DK, (int)tt, bar_raw);
        tma_load_2d(sm + R_K, &maps.k, hh * DK, (int)tt, bar_raw);
        tma_load_2d(sm + R_Q, &maps.q, hh * DK, (int)tt, bar_raw);
        if (!drop) tma_load_2d(sm + R_V, &maps.v, hh * DV, (int)tt, bar_raw);
    };

    int64_t item = next_valid(blockIdx.x);
    bool raw_in_flight = false;
    // beta of the next item, loaded one item ahead by threads < 64
    // raw bits of the next item's beta (bf16 in the low half, or fp32), converted when
    // used so that no instruction waits for the load before then
    uint32_t beta_bits = 0;
    auto load_beta = [&](int64_t tt, int hh, int LL) {
        beta_bits = 0;
        if (tid < LL) {
            const size_t idx = (size_t)(tt + tid) * H + hh;
            if constexpr (IN_BF16) beta_bits = __ldg(reinterpret_cast<const unsigned short*>(a.beta) + idx);
            else beta_bits = __float_as_uint(__ldg(reinterpret_cast<const float*>(a.beta) + idx));
        }
    };
    // the next item of this CTA after `from`, published in s_next by the last thread (it
    // is looked up one item ahead, while that thread idles in the triangular inverse)
    auto lookup_next = [&](int64_t from) {
        const int64_t nx = next_valid(from);
        int hh = 0, LL = 0;
        int64_t tt = 0;
        if (nx < n_items) item_info(a, nx, hh, tt, LL);
        s_next64[0] = nx;
        s_next64[1] = tt;
        s_next32[0] = hh;
        s_next32[1] = LL;
    };
    if (item < n_items) {
        int hh, LL;
        int64_t tt;
        item_info(a, item, hh, tt, LL);
        if (tid < CH) load_beta(tt, hh, LL);
        if constexpr (IN_BF16) {
            if (tid == 0) issue_raw(hh, tt, a.drop_tile && blockIdx.x == 0);
            raw_in_flight = true;
        }
    }
    if (tid == INTRA_THREADS - 1) lookup_next(item + gridDim.x);
    __syncthreads();

    while (item < n_items) {
        int h, L;
        int64_t t0;
        item_info(a, item, h, t0, L);
        uint8_t* wslot = a.ws + (size_t)item * SLOT_BYTES;
        const size_t rowstride = (size_t)H * DK;
        const size_t ebase = ((size_t)t0 * H + h) * DK + c;
        const size_t vbase = ((size_t)t0 * H + h) * DV + c;

        if (tid < CH) s_beta[tid] = IN_BF16 ? __uint_as_float(beta_bits << 16) : __uint_as_float(beta_bits);
        if constexpr (IN_BF16) {
            // a tile load that never completes ends the CTA's work, on every thread at once
            const bool ok = mbar_wait(bar_raw, ph_raw, a.status, a.wait_ns);
            if (__syncthreads_or(!ok)) break;
            ph_raw ^= 1;
            raw_in_flight = false;
        }

        // ---- a1: cumulative clamped log-decay g of this thread's tile (registers)
        float E1[16], E3[16];
        uint32_t qr2[8];  // raw q of this thread's 16 tokens, bf16 pairs (kept for the Qp epilogue)
        uint32_t kr2[8];  // raw k (bf16 inputs), kept from phase 1 for phase 2
        float G[5];
        {
            float alpha[16];
            float run = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = 16 * q4 + u;
                const float l = raw_in<IN_BF16>(sm, R_LA, a.log_alpha, ebase, rowstride, t, c, L);
                const float lc = (t < L) ? fmaxf(l, LOG_ALPHA_FLOOR) : 0.f;
                run += lc;
                alpha[u] = __expf(lc);  // per-step decay (1 past the end)
            }
            s_tot[q4 * 128 + c] = run;
            // E1 = e^{g_t - G_q4} = prod_{r<=t} alpha_r (<= 1),  E3 = e^{G_{q4+1} - g_t} = prod_{r>t} alpha_r
            // (products of at most 16 factors >= e^-5: no underflow in fp32)
            E1[0] = alpha[0];
#pragma unroll
            for (int u = 1; u < 16; ++u) E1[u] = E1[u - 1] * alpha[u];
            E3[15] = 1.f;
#pragma unroll
            for (int u = 14; u >= 0; --u) E3[u] = E3[u + 1] * alpha[u + 1];
            __syncthreads();
            float off = 0.f;
#pragma unroll
            for (int qq = 0; qq < 3; ++qq)
                if (qq < q4) off += s_tot[qq * 128 + c];
            // G_0 = 0, G_{b+1} = g at the last token of tile b
            s_G[(q4 + 1) * 128 + c] = off + run;
            if (q4 == 0) s_G[c] = 0.f;
            if (tid == 0) bulk_wait_read_all();  // previous item's slot copies have left X and Z2
            __syncthreads();
#pragma unroll
            for (int b = 0; b < 5; ++b) G[b] = s_G[b * 128 + c];
        }
        const float Gs = (q4 == 0) ? G[0] : (q4 == 1) ? G[1] : (q4 == 2) ? G[2] : G[3];  // G_q4
        const float Gn = (q4 == 0) ? G[1] : (q4 == 1) ? G[2] : (q4 == 2) ? G[3] : G[4];  // G_{q4+1}

        // ---- a2 operands (MN-major images, one 16-byte row = 8 consecutive tokens of channel c):
        //      KQr = [K o E1 ; scale Q o E1],  Kd = K o e^{G_q4 - g},  Kb^(b) = K o e^{G_b - g}  (b > q4)
        {
            const float eD = __expf(Gs - Gn);  // e^{G_q4 - G_{q4+1}} in [1, e^80]
            // factors e^{G_b - G_{q4+1}} for b = q4+1 .. 3 (the first is 1)
            const float f2 = __expf(((q4 == 0) ? G[2] : G[3]) - Gn);  // b = q4 + 2 (q4 <= 1)
            const float f3 = __expf(G[3] - Gn);                         // b = 3
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int tf = 16 * q4 + 8 * m;  // first token of this 8-token row
                float kr[8], qe[8], kd[8], k3[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = 8 * m + e, t = tf + e;
                    float kv, qv;
                    if constexpr (IN_BF16) {  // keep the raw bits (exact) for later phases
                        const uint32_t kb = raw_bits(sm, R_K, t, c, L), qb = raw_bits(sm, R_Q, t, c, L);
                        kv = __uint_as_float(kb << 16);
                        qv = __uint_as_float(qb << 16);
                        if (e & 1) {
                            kr2[u >> 1] |= kb << 16;
                            qr2[u >> 1] |= qb << 16;
                        } else {
                            kr2[u >> 1] = kb;
                            qr2[u >> 1] = qb;
                        }
                    } else {
                        kv = raw_in<IN_BF16>(sm, R_K, a.k, ebase, rowstride, t, c, L);
                        qv = raw_in<IN_BF16>(sm, R_Q, a.q, ebase, rowstride, t, c, L);
                        if (e & 1) qr2[u >> 1] |= (uint32_t)f32_to_bf16(qv) << 16;
                        else qr2[u >> 1] = (uint32_t)f32_to_bf16(qv);
                    }
                    kr[e] = kv * E1[u];
                    qe[e] = qv * E1[u] * a.scale;
                    k3[e] = kv * E3[u];
                    kd[e] = k3[e] * eD;  // k e^{G_q4 - g_t}, <= e^80
                }
                *reinterpret_cast<uint4*>(sm + IX_KQR + mn_off(tf, c, 2048)) = pack8(kr);
                *reinterpret_cast<uint4*>(sm + IX_KQR + mn_off(tf + 64, c, 2048)) = pack8(qe);
                *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(tf, c, KC_KG)) = pack8(kd);
                float f[8];
                if (q4 == 0) {
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B1 + tf, c, KC_KG)) = pack8(k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = k3[e] * f2;
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B2 + tf, c, KC_KG)) = pack8(f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = k3[e] * f3;
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B3 + tf, c, KC_KG)) = pack8(f);
                } else if (q4 == 1) {
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B2 + tf, c, KC_KG)) = pack8(k3);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = k3[e] * f3;
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B3 + tf, c, KC_KG)) = pack8(f);
                } else if (q4 == 2) {
                    *reinterpret_cast<uint4*>(sm + IX_KC + mn_off(KC_B3 + tf, c, KC_KG)) = pack8(k3);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- stage 1: [Kr;Qr] Kd^T and [Kr;Qr] Kb(b)^T
        if (tid == 0) {
            // one N = 160 product: [A/P diag | tile-1 | tile-2 | tile-3 off-diagonal] columns
            mma_mn<8, 2048, KC_KG>(tm + TM_AD, sb + IX_KQR, sb + IX_KC, idesc_bf16_major(128, 160, 1, 1));
            mma_commit(bar_mma);
        }

        // ---- phase 2 operands while stage 1 runs (K = token, own region Z2):
        //      KGt = (K o Gam)^T, Vt = V^T, Ktt = Kt^T
        {
            const float eG = __expf(Gs);          // Gam_t = E1 e^{G_q4}
            const float eC = __expf(G[4] - Gn);   // e^{g_C - g_t} = E3 e^{G_4 - G_{q4+1}}
#pragma unroll
            for (int m = 0; m < 2; ++m) {  // 8 consecutive tokens per 16-byte chunk
                float kg[8], vv[8], kt[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = 8 * m + e;
                    const int t = 16 * q4 + u;
                    float kv;
                    if constexpr (IN_BF16)
                        kv = __uint_as_float((u & 1) ? (kr2[u >> 1] & 0xFFFF0000u) : (kr2[u >> 1] << 16));
                    else
                        kv = raw_in<IN_BF16>(sm, R_K, a.k, ebase, rowstride, t, c, L);
                    vv[e] = raw_in<IN_BF16>(sm, R_V, a.v, vbase, (size_t)H * DV, t, c, L);
                    kg[e] = kv * E1[u] * eG;
                    kt[e] = kv * E3[u] * eC;
                }
                const uint32_t off = sw128_off((uint32_t)c, (uint32_t)(16 * q4 + 8 * m));
                *reinterpret_cast<uint4*>(sm + Z2_KGT + off) = pack8(kg);
                *reinterpret_cast<uint4*>(sm + Z2_VT + off) = pack8(vv);
                *reinterpret_cast<uint4*>(sm + Z2_KTT + off) = pack8(kt);
            }
        }
        __syncthreads();  // every read of RAW for this item is done
        // next item's raw tiles and beta
        const int64_t next = s_next64[0];
        if (next < n_items) {
            const int64_t tt = s_next64[1];
            const int hh = s_next32[0], LL = s_next32[1];
            if constexpr (IN_BF16) {
                if (tid == 0) issue_raw(hh, tt, false);
                raw_in_flight = true;
            }
            if (tid < CH) load_beta(tt, hh, LL);
        }
        mbar_wait_spin(bar_mma, ph_mma, a.status);
        ph_mma ^= 1;
        tc_fence_after();

        // ---- A (rows 0..63) -> fp32 smem [64][68];  P (rows 64..127) -> bf16 image Ph [t][s].
        //      Warp (qd, p): 16-column piece p of the 32 rows of quadrant qd.
        {
            float* sA = reinterpret_cast<float*>(sm + IY_A);
            const int p = q4;
            const int r = 32 * qd + lane;
            const bool isP = r >= 64;
            const int t = r & 63, bt = t >> 4;
            float dA[16], dB[16], dC[16];
            tmem_ld16(lane_addr + TM_AD + 16 * p, dA);
            if ((qd & 1) == 0) {
                if (p == 0) tmem_ld16(lane_addr + TM_B1, dB);  // rows of tile 1
            } else {
                if (p < 2) tmem_ld16(lane_addr + TM_B2 + 16 * p, dB);  // rows of tile 2
                if (p < 3) tmem_ld16(lane_addr + TM_B3 + 16 * p, dC);  // rows of tile 3
            }
            tmem_ld_wait();
            float d[16];
            bool write = true;
            if (p >= bt) {  // diagonal tile (A strictly lower, P lower) and the zero upper part
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) {
                    const int s = 16 * p + s16;
                    const bool keep = (p == bt) && (isP ? (s <= t) : (s < t));
                    d[s16] = keep ? dA[s16] : 0.f;
                }
            } else if (bt == 3) {
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) d[s16] = dC[s16];
            } else if (bt == 1 || bt == 2) {
#pragma unroll
                for (int s16 = 0; s16 < 16; ++s16) d[s16] = dB[s16];
            } else {
                write = false;
            }
            if (write) {
                if (isP) {
                    *reinterpret_cast<uint4*>(sm + IX_PH + sw128_off(t, 16 * p)) = pack8(d);
                    *reinterpret_cast<uint4*>(sm + IX_PH + sw128_off(t, 16 * p + 8)) = pack8(d + 8);
                } else {  // N = Diag(beta) A for the inverse
                    const float bt_ = s_beta[t];
                    float4* dst = reinterpret_cast<float4*>(sA + t * LDA + 16 * p);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_float4(bt_ * d[4 * i], bt_ * d[4 * i + 1], bt_ * d[4 * i + 2], bt_ * d[4 * i + 3]);
                }
            }
        }
        __syncthreads();

        // ---- a3: T = (I + N)^-1 Diag(beta) with N = Diag(beta) A (scaled when A was
        //      extracted), fp32, blocked on 16x16 tiles: X = (I + N)^-1 is built in sX from
        //      (1) the four 16x16 diagonal blocks by forward substitution, (2) the
        //      sub-diagonal blocks of the two 32x32 diagonal halves, X_{b+1,b} =
        //      -X_{b+1,b+1} N_{b+1,b} X_bb (b = 0, 2), (3) the lower-left 32x32 block
        //      X_LL = -H_1 N_LL H_0 (H_0, H_1 the halves).  Blocks above the diagonal are
        //      never read: the sums skip them and the T image writes zeros there.
        {
            const float* sA = reinterpret_cast<const float*>(sm + IY_A);
            float* sX = reinterpret_cast<float*>(sm + IY_X);
            float* sY = reinterpret_cast<float*>(sm + IX_TMP);  // partial products (8 KB)
            // idle here: look up the item after the next one (every thread read s_next at the
            // prefetch, before the extraction barrier)
            if (tid == INTRA_THREADS - 1) lookup_next(next + gridDim.x);
            float* sP = reinterpret_cast<float*>(sm + IY_A);  // [16][32], in the dead N region
            tri_inverse64(sA, sX, sY, sP, tid);
            {  // T = X Diag(beta) -> bf16 image Ti [t][s], 8 s per store, one row piece per thread
                const int t = tid >> 3, s0 = (tid & 7) * 8;
                float v8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if ((s0 >> 4) <= (t >> 4)) {
                    float4 x0 = *reinterpret_cast<const float4*>(sX + t * LDA + s0);
                    float4 x1 = *reinterpret_cast<const float4*>(sX + t * LDA + s0 + 4);
                    if (t >= 48 && s0 < 32) {  // the second half of block 3's lower-left sums
                        const float4 p0 = *reinterpret_cast<const float4*>(sP + (t - 48) * 32 + s0);
                        const float4 p1 = *reinterpret_cast<const float4*>(sP + (t - 48) * 32 + s0 + 4);
                        x0.x += p0.x; x0.y += p0.y; x0.z += p0.z; x0.w += p0.w;
                        x1.x += p1.x; x1.y += p1.y; x1.z += p1.z; x1.w += p1.w;
                    }
                    const float4 b0 = *reinterpret_cast<const float4*>(s_beta + s0);
                    const float4 b1 = *reinterpret_cast<const float4*>(s_beta + s0 + 4);
                    v8[0] = x0.x * b0.x; v8[1] = x0.y * b0.y; v8[2] = x0.z * b0.z; v8[3] = x0.w * b0.w;
                    v8[4] = x1.x * b1.x; v8[5] = x1.y * b1.y; v8[6] = x1.z * b1.z; v8[7] = x1.w * b1.w;
                }
                *reinterpret_cast<uint4*>(sm + IX_TI + sw128_off(t, s0)) = pack8(v8);
            }
        }

        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- stage 2: Wt = KGt Ti^T, Ut = Vt Ti^T
        if (tid == 0) {
            mma_sw128<4, 128, 64>(tm + TM_WT, sdesc_k_sw128(sb + Z2_KGT), sdesc_k_sw128(sb + IX_TI), idesc_bf16(128, 64));
            mma_sw128<4, 128, 64>(tm + TM_UT, sdesc_k_sw128(sb + Z2_VT), sdesc_k_sw128(sb + IX_TI), idesc_bf16(128, 64));
            mma_commit(bar_mma);
        }
        mbar_wait_spin(bar_mma, ph_mma, a.status);
        ph_mma ^= 1;
        tc_fence_after();
        {
            // group 0/1 -> Wt token columns [0,32)/[32,64), group 2/3 -> Ut; row = channel c
            const uint32_t col0 = (q4 < 2 ? TM_WT : TM_UT) + 32 * (q4 & 1);
            const uint32_t dst = q4 < 2 ? IY_WT : IY_UT;
            float d[32];
            tmem_ld16(lane_addr + col0, d);
            tmem_ld16(lane_addr + col0 + 16, d + 16);
            tmem_ld_wait();
#pragma unroll
            for (int pp = 0; pp < 4; ++pp)
                *reinterpret_cast<uint4*>(sm + dst + sw128_off((uint32_t)c, 32 * (q4 & 1) + 8 * pp)) = pack8(d + 8 * pp);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- stage 3: [Mlr | Bm] = Ktt [Wt ; Ut]^T (Wt and Ut are one 256-row image), then
        //      (P W)^T = Wt Ph^T and Ob = Ph Ut^T (M = 64) under a second commit, so that staging of
        //      Mlr and Bm overlaps the second pair of products.
        if (tid == 0) {
            const uint64_t dk = sdesc_k_sw128(sb + Z2_KTT), dw = sdesc_k_sw128(sb + IY_WT),
                           du = sdesc_k_sw128(sb + IY_UT), dp = sdesc_k_sw128(sb + IX_PH);
            mma_sw128<4, 128, 256>(tm + TM_M, dk, dw, idesc_bf16(128, 256));
            mma_commit(bar_mma);
            mma_sw128<4, 128, 64>(tm + TM_PW, dw, dp, idesc_bf16(128, 64));
            mma_sw128<4, 64, 128>(tm + TM_OB, dp, du, idesc_bf16(64, 128));
            mma_commit(bar_mma2);
        }
        // The slot is assembled in two shared-memory pieces that match its layout:
        // [Mlr | Qp | GamC] at IX (KQr/KC/Ti are dead) and [Bm | Ob] at Z2 (dead once
        // the first product is done); each leaves by one bulk copy.
        mbar_wait_spin(bar_mma, ph_mma, a.status);
        ph_mma ^= 1;
        tc_fence_after();
        {
            if (q4 < 2) {
                // Mlr row c, K block q4 -> K-major SW128 image
                uint8_t* dstM = sm + IX + SO_M + (size_t)q4 * (DK * 128);
#pragma unroll
                for (int hp = 0; hp < 2; ++hp) {
                    float d[32];
                    tmem_ld16(lane_addr + TM_M + 64 * q4 + 32 * hp, d);
                    tmem_ld16(lane_addr + TM_M + 64 * q4 + 32 * hp + 16, d + 16);
                    tmem_ld_wait();
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp)
                        *reinterpret_cast<uint4*>(dstM + sw128_off((uint32_t)c, (uint32_t)(32 * hp + 8 * pp))) =
                            pack8(d + 8 * pp);
                }
            } else {
                // Bm row c, value columns [64 (q4-2), +64) -> slices 2 (q4-2) and 2 (q4-2) + 1
                const int hh = q4 - 2;
#pragma unroll
                for (int hp = 0; hp < 2; ++hp) {  // one 32-column slice per half
                    float d[32];
                    tmem_ld16(lane_addr + TM_BM + 64 * hh + 32 * hp, d);
                    tmem_ld16(lane_addr + TM_BM + 64 * hh + 32 * hp + 16, d + 16);
                    tmem_ld_wait();
                    uint4* dstB = reinterpret_cast<uint4*>(sm + Z2 + (size_t)(2 * hh + hp) * BSL + (size_t)c * DVS * 2);
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp) dstB[swz64(c, pp)] = pack8(d + 8 * pp);
                }
                if (q4 == 3) *reinterpret_cast<float*>(sm + IX + SO_G + 4 * c) = __expf(G[4]);  // Gam_C
            }
        }
        // Mlr and Bm leave now, so that the bulk-copy engine is free earlier for the next
        // item's tile loads; Qp, GamC and Ob follow at the end of the item
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(wslot + SO_M, sm + IX + SO_M, (uint32_t)(SO_Q - SO_M));
            bulk_s2g(wslot + SO_B, sm + Z2, (uint32_t)(SO_O - SO_B));
            bulk_commit();
        }
        mbar_wait_spin(bar_mma2, ph_mma2, a.status);
        ph_mma2 ^= 1;
        tc_fence_after();
        {
            // Qp^T[c][t] = scale q_tc e^{g_tc} - (P W)^T[c][t] -> MN-major image (token-contiguous
            // rows), this thread's 16 tokens
            const float eG = __expf(Gs);
            float pw[16], qq[16];
            tmem_ld16(lane_addr + TM_PW + 16 * q4, pw);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float qv = __uint_as_float((u & 1) ? (qr2[u >> 1] & 0xFFFF0000u) : (qr2[u >> 1] << 16));
                qq[u] = qv * E1[u] * eG * a.scale - pw[u];
            }
            const int tf = 16 * q4;
            uint8_t* dstQ = sm + IX + SO_Q;
            *reinterpret_cast<uint4*>(dstQ + mn_off(tf, c, 1024)) = pack8(qq);
            *reinterpret_cast<uint4*>(dstQ + mn_off(tf + 8, c, 1024)) = pack8(qq + 8);
        }
        {
            // Ob row t = 16 qd + lane (lanes < 16 of each quadrant), value slice q4 -> [slice][t][32]
            float ob[32];
            tmem_ld16(lane_addr + TM_OB + 32 * q4, ob);
            tmem_ld16(lane_addr + TM_OB + 32 * q4 + 16, ob + 16);
            tmem_ld_wait();
            if (lane < 16) {
                uint4* dstO = reinterpret_cast<uint4*>(sm + Z2 + (SO_O - SO_B) + (size_t)q4 * OSL +
                                                       (size_t)(16 * qd + lane) * (DVS * 2));
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) dstO[swz64(16 * qd + lane, pp)] = pack8(ob + 8 * pp);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            bulk_s2g(wslot + SO_Q, sm + IX + SO_Q, (uint32_t)(SO_MQG - SO_Q));  // Qp + GamC
            bulk_s2g(wslot + SO_O, sm + Z2 + (SO_O - SO_B), (uint32_t)(SLOT_BYTES - SO_O));
            bulk_commit();
        }
        item = next;
    }
    // tile loads can only be in flight here after a failed wait; let them land (bounded)
    if constexpr (IN_BF16) {
        if (tid == 0 && raw_in_flight) mbar_wait(bar_raw, ph_raw, nullptr, a.wait_ns);
    }
    if (tid == 0) bulk_wait_all();  // last slot copy complete before the CTA retires
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, INTRA_TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// chain_kernel
// ---------------------------------------------------------------------------
// One CTA per (sequence, head, 32-column value slice), warp-specialised:
//   warps 0-3 (consumers): thread c owns state row c of the slice (32 fp32
//     registers); applies S <- GamC o S - Mlr S + Bm, writes the next bf16
//     state operand image, then forms the chunk output o = Qp S + Ob;
//   warp 4 (one thread): the tensor-core products Mlr S and Qp S;
//   warp 5 (one thread): bulk loads of the chunk operands, three chunks ahead,
//     into buffers the consumers release as soon as they hold their Ob row
//     and gate columns in registers.
// The roles meet only on mbarriers, so the issue of the next products
// overlaps the output work of the current chunk and never waits for a refill.  TMEM (128 columns): D_S =
// Mlr S in [0,32) (M=128, lane = row c); D_O = Qp S double-buffered in [32,64)
// and [64,96) (M=64: row t lives in lane 32*(t/16) + t%16).  Shared memory:
// three chunk buffers {Mlr image 32K, Qp image 16K, GamC 512, Bm slice 8K, Ob
// slice [64 tokens][32 cols] 4K[, gate tile 4K]} and two bf16 state operand
// images (MN-major without swizzle: value columns contiguous, 8 KB each).
//
// Barriers and the order that keeps each phase from being skipped:
//   bar_img   consumers (128) -> producer: state image of chunk i written.  The
//             image of chunk i + 1 is written after D_S(i) is read, i.e. after
//             the producer issued chunk i.
//   bar_s     commit of Mlr S(i); it also covers Qp S(i - 1), so the image
//             that product read may be rewritten once bar_s(i) is seen.
//   bar_o[2]  commit of Qp S(i) into D_O[i & 1]; D_O[i & 1] is overwritten by
//             chunk i + 2, issued after the image of i + 2, which consumers
//             write after reading D_O(i).
//   bar_ld[3] loads of a buffer; bar_free[3] consumers (128) -> loader: the
//             buffer is no longer read (the products that read it completed:
//             the consumer saw bar_o of its chunk first) and may be refilled.
//
// With the fused gate (GATE), the four CTAs of one (sequence, head) -- its four
// value-column slices -- form a thread-block cluster.  The per-head RMSNorm
// needs sum_j o_tj^2 over all 128 columns: each CTA pushes its 64 per-row
// partial sums into every CTA's shared memory (distributed shared memory) with
// asynchronous stores that count down a transaction barrier in the receiving
// CTA; the normalisation of chunk i is finished during iteration i + 1.
// Reuse of the two partial-sum slots: a peer writes row t of slot i & 1 for
// chunk i + 2 only after it has received every CTA's chunk-(i + 1) partials,
// and this CTA's row-t thread sends its chunk-(i + 1) partial after it has read
// row t of the chunk-i slot.
constexpr uint32_t CB_M = 0, CB_Q = 32768, CB_G = 49152, CB_B = 49664, CB_O = 57856, CB_GT = 61952;
constexpr int NBUF = 3;  // chunk buffers in flight
template <bool GATE> struct ChainLayout {
    static constexpr uint32_t CB_SIZE = GATE ? 66560u : 62464u;  // multiples of 1024
    static constexpr uint32_t SB = NBUF * CB_SIZE;                // two 8K state images
    static constexpr uint32_t PART = SB + 2 * 8192;               // [2][4 slices][64 rows] fp32
    static constexpr uint32_t BAR = PART + (GATE ? 2048u : 0u);   // barriers (128 B)
    static constexpr uint32_t TMEMP = BAR + 128;
    static constexpr uint32_t SMEM = TMEMP + 16 + 1024;
};
constexpr uint32_t CHAIN_TMEM_COLS = 128;
constexpr uint32_t SB_KG = DVS * 16;  // state image K-group stride: 8 key rows x 32 columns x 2 B
constexpr int CHAIN_THREADS = 192;  // 4 consumer warps + 1 tensor-issue warp + 1 loader warp
constexpr int CLUSTER = NSL;        // CTAs per (sequence, head) when the gate is fused
constexpr uint32_t PART_TX = CLUSTER * 64 * 4;  // partial-sum bytes each CTA receives per chunk

// SEG = 0: the plain walk over this pass's chunks.  Segment-parallel prefill (each
// sequence cut into a.segs segments of whole chunks, blockIdx.z = n * segs + g):
//   (pass 1, each segment's affine map, is map_walk_kernel's)
// SEG = 2: segment g first folds segments 0 .. g-1 into the initial state through
//   their slots, then walks its own chunks with outputs; the last segment writes
//   the final state;
// SEG = 3: the plain walk without outputs, keeping only the states (checkpoints
//   and the final state): the forward recomputation of the backward pass.
template <bool OUT_BF16, bool GATE, int SEG>
__global__ void __launch_bounds__(CHAIN_THREADS, 1)
chain_kernel(const ChunkArgs a, const __grid_constant__ CUtensorMap gate_map, const float* __restrict__ norm_w,
             float eps) {
    using LY = ChainLayout<GATE>;
    constexpr uint32_t CB_SIZE = LY::CB_SIZE;
    if (a.wait_first) pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool consumer = warp < 4;
    const int js = blockIdx.x, h = blockIdx.y;
    const int n = SEG == 2 ? (int)blockIdx.z / a.segs : (int)blockIdx.z;
    const int g = SEG == 2 ? (int)blockIdx.z % a.segs : 0;
    const int H = a.H;
    const int jb = js & (NSL - 1);                // value slice of Bm / outputs
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + LY::BAR);         // [NBUF]
    uint64_t* bar_free = reinterpret_cast<uint64_t*>(sm + LY::BAR + 24);  // [NBUF]
    uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + LY::BAR + 48);
    uint64_t* bar_o = reinterpret_cast<uint64_t*>(sm + LY::BAR + 56);     // [2]
    uint64_t* bar_img = reinterpret_cast<uint64_t*>(sm + LY::BAR + 72);
    uint64_t* bar_part = reinterpret_cast<uint64_t*>(sm + LY::BAR + 80);  // [2], gate only
    float* s_part = reinterpret_cast<float*>(sm + LY::PART);              // [2][4][64], gate only
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + LY::TMEMP);

    int64_t s_beg, s_end;
    seq_range(a, n, s_beg, s_end);
    const int nchunks = (int)((s_end - s_beg + CH - 1) / CH);
    // chunk iterations [c_beg, c_end); with SEG = 2 preceded by nseg segment iterations
    int c_beg, c_end;
    if constexpr (SEG == 0 || SEG == 3) {
        c_beg = a.i0;
        c_end = min(a.i0 + a.wc, nchunks);
    } else {
        const int per = (nchunks + a.segs - 1) / a.segs;
        c_beg = min(g * per, nchunks);
        c_end = min(c_beg + per, nchunks);
    }
    const int nseg = SEG == 2 ? g : 0;
    const int nck = c_end > c_beg ? c_end - c_beg : 0;
    const int nit = nseg + nck;  // the same for the whole cluster

    // state slice: row tid, columns [32 jb, 32 jb + 32)
    const size_t st_off = (((size_t)n * H + h) * DK + (consumer ? tid : 0)) * DV + (size_t)DVS * jb;
    float S[DVS];
    if (consumer) {
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
            for (int i = 0; i < NBUF; ++i) {
                mbar_init(&bar_ld[i], 1);
                mbar_init(&bar_free[i], 128);
            }
            mbar_init(bar_s, 1);
            mbar_init(&bar_o[0], 1);
            mbar_init(&bar_o[1], 1);
            mbar_init(bar_img, 128);
            if constexpr (GATE) {
                // one local arrival (with the byte count) plus 4 B from every row of every CTA per chunk
                mbar_init(&bar_part[0], 1);
                mbar_init(&bar_part[1], 1);
                mbar_arrive_expect_tx(&bar_part[0], PART_TX);
                mbar_arrive_expect_tx(&bar_part[1], PART_TX);
            }
            fence_mbar_init();
        }
        __syncthreads();
        if constexpr (GATE) cluster_sync_all();  // peers' barriers exist before any remote store
        tc_fence_after();
        pdl_wait();  // the slots (and segment slots) written by the kernel ahead of this one
        const uint32_t tm = *s_tmem;
        const size_t slot0 = ((size_t)n * a.wc + (c_beg - a.i0)) * H + h;  // slot of the first chunk iteration
        // iteration it: a segment iteration (it < nseg) or chunk c_beg + it - nseg;
        // only chunk iterations of SEG != 1 form outputs (output index oi = it - nseg)
        auto slot_of = [&](int it) -> const uint8_t* {
            if (SEG == 2 && it < nseg) return a.seg_ws + (((size_t)n * a.segs + it) * H + h) * SLOT_BYTES;
            return a.ws + (slot0 + (size_t)(it - nseg) * H) * SLOT_BYTES;
        };
        auto has_out = [&](int it) { return SEG != 1 && SEG != 3 && it >= nseg; };
        // chunk buffer of iteration it and its barrier phase
        auto bidx = [](int it) { return it % NBUF; };
        auto bpar = [](int it) { return (uint32_t)((it / NBUF) & 1); };
        bool failed = false;
        // loader / issuer bookkeeping for the bounded drain
        int loads_issued = 0, mma_issued = 0;

        if (warp == 5) {
            // -------------------------------------------------------- loader
            // (its own warp, so that waiting for a buffer to be released never holds up the
            // tensor-core issue)
            if (lane == 0) {
                auto issue_load = [&](int it) {
                    const int b = bidx(it);
                    uint8_t* buf = sm + b * CB_SIZE;
                    const uint8_t* src = slot_of(it);
                    const bool out = has_out(it);
                    mbar_arrive_expect_tx(&bar_ld[b], SO_MQG + BSL + (out ? OSL + (GATE ? (uint32_t)(CH * DVS * 2) : 0u) : 0u));
                    bulk_g2s(buf + CB_M, src + SO_M, SO_MQG, &bar_ld[b]);
                    bulk_g2s(buf + CB_B, src + SO_B + (size_t)jb * BSL, BSL, &bar_ld[b]);
                    if (out) {
                        bulk_g2s(buf + CB_O, src + SO_O + (size_t)jb * OSL, OSL, &bar_ld[b]);
                        if constexpr (GATE)  // gate tile [64 tokens][32 value cols] of this slice, 64-byte swizzled
                            tma_load_2d(buf + CB_GT, &gate_map, h * DV + DVS * jb,
                                        (int)(s_beg + (int64_t)(c_beg + it - nseg) * CH), &bar_ld[b]);
                    }
                };
                for (int j = 0; j < NBUF && j < nit; ++j) {
                    issue_load(j);
                    loads_issued = j + 1;
                }
                // chunk r = j + NBUF goes into the buffer of chunk j once the consumers released it
                for (int j = 0; j + NBUF < nit; ++j) {
                    if (!mbar_wait(&bar_free[bidx(j)], bpar(j), a.status)) {
                        failed = true;
                        break;
                    }
                    issue_load(j + NBUF);
                    loads_issued = j + NBUF + 1;
                }
            }
        } else if (warp == 4) {
            // -------------------------------------------------- tensor issue
            if (lane == 0) {
                for (int it = 0; it < nit; ++it) {
                    const int b = bidx(it);
                    if (!mbar_wait_spin(bar_img, (uint32_t)(it & 1), a.status) ||
                        !mbar_wait_spin(&bar_ld[b], bpar(it), a.status)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    // Mlr S -> D_S, then Qp S -> D_O[it & 1]
                    // state image: MN-major, K-group (8 key rows) stride SB_KG, 8-column block stride 128
                    const uint64_t sdesc = sdesc_interleave(sbase + LY::SB + (it & 1) * 8192, SB_KG, 128u);
                    {  // Mlr (K-major SW128) x state image
                        const uint64_t mdesc = sdesc_k_sw128(sbase + b * CB_SIZE + CB_M);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            mma_bf16(tm + 0, mdesc + (uint32_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4),
                                     sdesc + (uint32_t)((kk * 2 * SB_KG) >> 4), idesc_bf16_major(128, DVS, 0, 1),
                                     kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_s);
                    if (has_out(it)) {  // Qp (MN-major, no swizzle) x state image -> D_O[oi & 1]
                        const int oi = it - nseg;
                        const uint64_t qdesc = sdesc_interleave(sbase + b * CB_SIZE + CB_Q, 1024u, 128u);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            mma_bf16(tm + 32 + 32 * (oi & 1), qdesc + (uint32_t)((kk * 2048) >> 4),
                                     sdesc + (uint32_t)((kk * 2 * SB_KG) >> 4), idesc_bf16_major(64, DVS, 1, 1),
                                     kk > 0 ? 1u : 0u);
                        mma_commit(&bar_o[oi & 1]);
                    }
                    mma_issued = it + 1;
                }
            }
        } else {
            // ----------------------------------------------------- consumers
            const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
            // bf16 state operand, MN-major without swizzle (value columns contiguous): key
            // row c's 32 columns are four 16-byte pieces, one per 8-column block
            auto write_state_image = [&](int it) {
                uint8_t* img = sm + LY::SB + (it & 1) * 8192 + ((uint32_t)tid >> 3) * SB_KG + ((uint32_t)tid & 7u) * 16u;
#pragma unroll
                for (int nb = 0; nb < DVS / 8; ++nb) *reinterpret_cast<uint4*>(img + nb * 128) = pack8(S + 8 * nb);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bar_img);
            };

            // output row served by this lane: lanes 0-15 hold it in TMEM (M = 64
            // layout); with the fused gate, lanes 16-31 take over its columns 16-31
            const int trow = 16 * warp + (lane & 15);
            const int hi = lane >> 4;
            constexpr int HC = DVS / 2;  // columns per lane in the gate epilogue
            float w16[GATE ? HC : 1];
            float o_prev[GATE ? HC : 1];
            uint32_t g_prev[GATE ? HC / 2 : 1];
            int64_t t0_prev = 0;
            int L_prev = 0;
            if constexpr (GATE) {
#pragma unroll
                for (int j = 0; j < HC; ++j) w16[j] = norm_w ? __ldg(norm_w + DVS * jb + HC * hi + j) : 1.0f;
            }
            // finishes y = o * rsqrt(mean o^2 + eps) * w * sigmoid(g) for output chunk itp
            auto finish_prev = [&](int itp) -> bool {
                if (!mbar_wait_cluster(&bar_part[itp & 1], (uint32_t)((itp >> 1) & 1), a.status)) return false;
                // arm the slot's barrier for chunk itp + 2 (its bytes may already be arriving)
                if (tid == 0 && itp + 2 < nck) mbar_arrive_expect_tx(&bar_part[itp & 1], PART_TX);
                if (trow < L_prev) {
                    const float* pp = s_part + (itp & 1) * (CLUSTER * 64);
                    float ss = 0.f;
#pragma unroll
                    for (int r = 0; r < CLUSTER; ++r) ss += pp[r * 64 + trow];
                    const float inv = rsqrtf(ss * (1.0f / DV) + eps);
                    const size_t obase = ((size_t)(t0_prev + trow) * H + h) * DV + (size_t)DVS * jb + HC * hi;
#pragma unroll
                    for (int m = 0; m < HC / 8; ++m) {
                        float y8[8];
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            const int j = 8 * m + p;
                            const float gj =
                                __uint_as_float((j & 1) ? (g_prev[j >> 1] & 0xFFFF0000u) : (g_prev[j >> 1] << 16));
                            y8[p] = o_prev[j] * inv * w16[j] * sigmoid_fast(gj);
                        }
                        if constexpr (OUT_BF16) {
                            reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.o) + obase)[m] = pack8(y8);
                        } else {
                            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + obase) + 2 * m;
                            dst[0] = make_float4(y8[0], y8[1], y8[2], y8[3]);
                            dst[1] = make_float4(y8[4], y8[5], y8[6], y8[7]);
                        }
                    }
                }
                return true;
            };

            // checkpoint: the state after (j + 1) * ckpt_every whole chunks of the sequence
            auto store_ckpt = [&](int oi) {
                if (!a.ckpt) return;
                const int cdone = c_beg + oi + 1;  // chunks of this sequence now folded in
                const int64_t t_end = s_beg + (int64_t)cdone * CH;
                if (cdone % a.ckpt_every == 0 && t_end <= s_end && cdone / a.ckpt_every <= a.n_ckpt) {
                    const int j = cdone / a.ckpt_every - 1;
                    if constexpr (SEG == 3) {
                        // the backward's chunk-boundary states: bf16 operand images (row tid, columns
                        // [32 jb, 32 jb + 32)), bulk-copied by its chunk-local kernel
                        uint8_t* img = reinterpret_cast<uint8_t*>(a.ckpt) +
                                       (((size_t)n * a.n_ckpt + j) * H + h) * STATE_IMG_BYTES;
#pragma unroll
                        for (int m = 0; m < DVS / 8; ++m)
                            *reinterpret_cast<uint4*>(img + state_img_off((uint32_t)tid, (uint32_t)(DVS * jb + 8 * m))) =
                                pack8(S + 8 * m);
                    } else {
                        float* dst = a.ckpt + ((((size_t)n * a.n_ckpt + j) * H + h) * DK + tid) * DV + (size_t)DVS * jb;
#pragma unroll
                        for (int c4 = 0; c4 < DVS; c4 += 4)
                            __stcs(reinterpret_cast<float4*>(dst + c4),
                                   make_float4(S[c4], S[c4 + 1], S[c4 + 2], S[c4 + 3]));
                    }
                }
            };

            write_state_image(0);
            for (int it = 0; it < nit; ++it) {
                const int b = bidx(it);
                const uint8_t* buf = sm + b * CB_SIZE;
                const int oi = it - nseg;  // output index (chunk iterations)
                const int64_t t0 = s_beg + (int64_t)(c_beg + oi) * CH;
                const int L = (int)((s_end - t0) < CH ? (s_end - t0) : CH);

                // (1) state update: S <- GamC o S - Mlr S + Bm
                if (!mbar_wait_spin(bar_s, (uint32_t)(it & 1), a.status) || !mbar_wait_spin(&bar_ld[b], bpar(it), a.status)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                {
                    float ds[DVS];
                    tmem_ld32(lane_addr + 0, ds);
                    tmem_ld_wait();
                    const float gamC = *reinterpret_cast<const float*>(buf + CB_G + 4 * tid);
                    const uint4* bsrc = reinterpret_cast<const uint4*>(buf + CB_B + (uint32_t)tid * DVS * 2);
#pragma unroll
                    for (int m = 0; m < DVS / 8; ++m) {
                        const uint4 w = bsrc[swz64(tid, m)];
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const int j = 8 * m + 2 * p;
                            const float b0 = __uint_as_float(ww[p] << 16);
                            const float b1 = __uint_as_float(ww[p] & 0xFFFF0000u);
                            S[j] = gamC * S[j] - ds[j] + b0;
                            S[j + 1] = gamC * S[j + 1] - ds[j + 1] + b1;
                        }
                    }
                }
                // (2) the next chunk's state operand (D_S has been read)
                if (it + 1 < nit) write_state_image(it + 1);
                if (!has_out(it)) {  // a segment iteration, or no outputs at all: the buffer is done
                    mbar_arrive(&bar_free[b]);
                    if constexpr (SEG == 3) store_ckpt(oi);
                    continue;
                }
                // (3) this chunk's output: o = Qp S + Ob  (then y, when the gate is fused)
                if (!mbar_wait_spin(&bar_o[oi & 1], (uint32_t)((oi >> 1) & 1), a.status)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float ov[DVS];
                {
                    float dO[DVS];
                    tmem_ld32(lane_addr + 32 + 32 * (oi & 1), dO);
                    tmem_ld_wait();
                    // Ob slice [64 tokens][32 value cols]: row trow
                    const uint4* orow = reinterpret_cast<const uint4*>(buf + CB_O + (uint32_t)trow * (DVS * 2));
#pragma unroll
                    for (int m = 0; m < DVS / 8; ++m) {
                        const uint4 w = orow[swz64(trow, m)];
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            ov[8 * m + 2 * p] = dO[8 * m + 2 * p] + __uint_as_float(ww[p] << 16);
                            ov[8 * m + 2 * p + 1] = dO[8 * m + 2 * p + 1] + __uint_as_float(ww[p] & 0xFFFF0000u);
                        }
                    }
                }
                uint32_t g_cur[GATE ? HC / 2 : 1];
                if constexpr (GATE) {  // this chunk's gate columns of the lane's row (64-byte swizzled tile)
                    const uint4* gsrc = reinterpret_cast<const uint4*>(buf + CB_GT + (uint32_t)trow * DVS * 2);
#pragma unroll
                    for (int m = 0; m < HC / 8; ++m) {
                        const uint4 w = gsrc[swz64(trow, 2 * hi + m)];
                        g_cur[4 * m] = w.x; g_cur[4 * m + 1] = w.y; g_cur[4 * m + 2] = w.z; g_cur[4 * m + 3] = w.w;
                    }
                }
                mbar_arrive(&bar_free[b]);  // everything this thread reads from the buffer is in registers
                if constexpr (!GATE) {
                    if (lane < 16 && trow < L) {
                        const size_t obase = ((size_t)(t0 + trow) * H + h) * DV + (size_t)DVS * jb;
#pragma unroll
                        for (int m = 0; m < DVS / 8; ++m) {
                            if constexpr (OUT_BF16) {
                                reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.o) + obase)[m] = pack8(ov + 8 * m);
                            } else {
                                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + obase) + 2 * m;
                                dst[0] = make_float4(ov[8 * m], ov[8 * m + 1], ov[8 * m + 2], ov[8 * m + 3]);
                                dst[1] = make_float4(ov[8 * m + 4], ov[8 * m + 5], ov[8 * m + 6], ov[8 * m + 7]);
                            }
                        }
                    }
                } else {
                    // finish the previous chunk first (its partials are read before this
                    // chunk's partials are published, which orders the slot reuse)
                    if (oi > 0 && !finish_prev(oi - 1)) {
                        failed = true;
                        break;
                    }
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        const float up = __shfl_up_sync(0xFFFFFFFFu, ov[HC + j], 16);
                        o_prev[j] = hi ? up : ov[j];
                        ss += o_prev[j] * o_prev[j];
                    }
                    ss += __shfl_down_sync(0xFFFFFFFFu, ss, 16);  // lanes 0-15: the whole 32-column row
#pragma unroll
                    for (int m = 0; m < HC / 2; ++m) g_prev[m] = g_cur[m];  // kept for the next iteration
                    if (lane < 16) {
                        const uint32_t slot = smem_u32(s_part + (oi & 1) * (CLUSTER * 64) + jb * 64 + trow);
                        const uint32_t barl = smem_u32(&bar_part[oi & 1]);
#pragma unroll
                        for (int r = 0; r < CLUSTER; ++r)
                            st_async_f32(map_to_cta(slot, (uint32_t)r), ss, map_to_cta(barl, (uint32_t)r));
                    }
                    t0_prev = t0;
                    L_prev = L;
                }
                store_ckpt(oi);
                // (4) D_O[oi & 1] is no longer read
                tc_fence_before();
            }
            if constexpr (GATE) {
                if (!failed && nck > 0 && !finish_prev(nck - 1)) failed = true;
            }
        }

        // copies and products still in flight finish before the CTA retires (bounded; in a
        // normal run every one of them has been consumed and the waits return at once):
        // the loader's last load into each buffer, the issuer's last pair of products
        __syncthreads();
        if (warp == 5 && lane == 0) {
            for (int j = loads_issued - NBUF < 0 ? 0 : loads_issued - NBUF; j < loads_issued; ++j)
                mbar_wait(&bar_ld[bidx(j)], bpar(j), nullptr);
        }
        if (warp == 4 && lane == 0 && failed && mma_issued > 0) {
            const int j = mma_issued - 1;
            mbar_wait(bar_s, (uint32_t)(j & 1), nullptr);
            if (has_out(j)) mbar_wait(&bar_o[(j - nseg) & 1], (uint32_t)(((j - nseg) >> 1) & 1), nullptr);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tm, CHAIN_TMEM_COLS);
        if constexpr (GATE) cluster_sync_all();  // no CTA leaves while a peer may still write to it
    }

    // the carried / final state slice (with segments: the last segment's)
    if (consumer && (SEG != 2 || g == a.segs - 1)) {
#pragma unroll
        for (int j = 0; j < DVS; j += 4)
            *reinterpret_cast<float4*>(a.state_io + st_off + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
}

// ---------------------------------------------------------------------------
// map_walk_kernel
// ---------------------------------------------------------------------------
// The affine map S -> M_g S + B_g of a segment of whole chunks (segment-parallel
// prefill, pass 1; the per-device step of context parallelism across devices): one CTA
// per (sequence and segment, head, 32-column slice jb) carries both the slice of B_g
// (the state walked from zero, with B_m) and the slice of M_g (the identity walked
// without B_m), so the chunk's one tensor-core product M_lr [S_B | S_M] has N = 64 and a
// head needs four CTAs.  Roles as in chain_kernel: warps 0-3 own one row each of both
// slices (64 fp32 registers), warp 4 issues the products, warp 5 bulk-loads each chunk's
// M_lr image, Gamma_C and B_m slice three chunks ahead.
constexpr uint32_t MW_M = 0, MW_G = 32768, MW_B = 33280;         // one chunk buffer
constexpr uint32_t MW_BUF = 41984;                               // 1024-aligned stride
constexpr uint32_t MW_IMG = NBUF * MW_BUF;                       // [S_B | S_M] bf16 image, 16 KB
constexpr uint32_t MW_BAR = MW_IMG + 16384;
constexpr uint32_t MW_TMEMP = MW_BAR + 128;
constexpr uint32_t MW_SMEM = MW_TMEMP + 16 + 1024;
constexpr uint32_t MW_KG = 2 * DVS * 16;  // image K-group (8 key rows) stride: 64 columns x 2 B x 8 rows

__global__ void __launch_bounds__(CHAIN_THREADS, 1) map_walk_kernel(const ChunkArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool consumer = warp < 4;
    const int jb = blockIdx.x, h = blockIdx.y;
    const int n = (int)blockIdx.z / a.segs, g = (int)blockIdx.z % a.segs;
    const int H = a.H;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + MW_BAR);         // [NBUF]
    uint64_t* bar_free = reinterpret_cast<uint64_t*>(sm + MW_BAR + 24);  // [NBUF]
    uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + MW_BAR + 48);
    uint64_t* bar_img = reinterpret_cast<uint64_t*>(sm + MW_BAR + 56);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + MW_TMEMP);

    int64_t s_beg, s_end;
    seq_range(a, n, s_beg, s_end);
    const int nchunks = (int)((s_end - s_beg + CH - 1) / CH);
    const int per = (nchunks + a.segs - 1) / a.segs;
    const int c_beg = min(g * per, nchunks), c_end = min(c_beg + per, nchunks);
    const int nit = c_end > c_beg ? c_end - c_beg : 0;

    // row tid: SB = columns [32 jb, +32) of B_g (from zero), SM = the same columns of M_g (from I)
    float SB[DVS], SM[DVS];
#pragma unroll
    for (int j = 0; j < DVS; ++j) {
        SB[j] = 0.f;
        SM[j] = (consumer && tid == DVS * jb + j) ? 1.f : 0.f;
    }
    if (nit > 0) {
        if (warp == 0) {
            tmem_alloc(s_tmem, 64);
            tmem_relinquish();
        }
        if (tid == 0) {
            for (int i = 0; i < NBUF; ++i) {
                mbar_init(&bar_ld[i], 1);
                mbar_init(&bar_free[i], 128);
            }
            mbar_init(bar_s, 1);
            mbar_init(bar_img, 128);
            fence_mbar_init();
        }
        __syncthreads();
        tc_fence_after();
        const uint32_t tm = *s_tmem;
        const size_t slot0 = ((size_t)n * a.wc + (c_beg - a.i0)) * H + h;
        auto slot_of = [&](int it) -> const uint8_t* { return a.ws + (slot0 + (size_t)it * H) * SLOT_BYTES; };
        auto bidx = [](int it) { return it % NBUF; };
        auto bpar = [](int it) { return (uint32_t)((it / NBUF) & 1); };
        bool failed = false;
        int loads_issued = 0, mma_issued = 0;

        if (warp == 5) {
            if (lane == 0) {
                auto issue_load = [&](int it) {
                    const int b = bidx(it);
                    uint8_t* buf = sm + b * MW_BUF;
                    const uint8_t* src = slot_of(it);
                    mbar_arrive_expect_tx(&bar_ld[b], 32768u + 512u + BSL);
                    bulk_g2s(buf + MW_M, src + SO_M, 32768u, &bar_ld[b]);
                    bulk_g2s(buf + MW_G, src + SO_G, 512u, &bar_ld[b]);
                    bulk_g2s(buf + MW_B, src + SO_B + (size_t)jb * BSL, BSL, &bar_ld[b]);
                };
                for (int j = 0; j < NBUF && j < nit; ++j) {
                    issue_load(j);
                    loads_issued = j + 1;
                }
                for (int j = 0; j + NBUF < nit; ++j) {
                    if (!mbar_wait(&bar_free[bidx(j)], bpar(j), a.status)) {
                        failed = true;
                        break;
                    }
                    issue_load(j + NBUF);
                    loads_issued = j + NBUF + 1;
                }
            }
        } else if (warp == 4) {
            if (lane == 0) {
                const uint32_t idesc = idesc_bf16_major(128, 2 * DVS, 0, 1);
                for (int it = 0; it < nit; ++it) {
                    const int b = bidx(it);
                    if (!mbar_wait_spin(bar_img, (uint32_t)(it & 1), a.status) ||
                        !mbar_wait_spin(&bar_ld[b], bpar(it), a.status)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t sdesc = sdesc_interleave(sbase + MW_IMG, MW_KG, 128u);
                    const uint64_t mdesc = sdesc_k_sw128(sbase + b * MW_BUF + MW_M);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        mma_bf16(tm, mdesc + (uint32_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4),
                                 sdesc + (uint32_t)((kk * 2 * MW_KG) >> 4), idesc, kk > 0 ? 1u : 0u);
                    mma_commit(bar_s);
                    mma_issued = it + 1;
                }
            }
        } else {
            const uint32_t lane_addr = tm + ((uint32_t)(32 * warp) << 16);
            // [S_B | S_M] as the bf16 B operand: MN-major without swizzle, key row tid's 64
            // columns as eight 16-byte pieces, one per 8-column block
            auto write_image = [&]() {
                uint8_t* img = sm + MW_IMG + ((uint32_t)tid >> 3) * MW_KG + ((uint32_t)tid & 7u) * 16u;
#pragma unroll
                for (int nb = 0; nb < DVS / 8; ++nb) {
                    *reinterpret_cast<uint4*>(img + nb * 128) = pack8(SB + 8 * nb);
                    *reinterpret_cast<uint4*>(img + (DVS / 8 + nb) * 128) = pack8(SM + 8 * nb);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bar_img);
            };
            write_image();
            for (int it = 0; it < nit; ++it) {
                const int b = bidx(it);
                const uint8_t* buf = sm + b * MW_BUF;
                if (!mbar_wait_spin(bar_s, (uint32_t)(it & 1), a.status) || !mbar_wait_spin(&bar_ld[b], bpar(it), a.status)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float d[DVS];
                const float gamC = *reinterpret_cast<const float*>(buf + MW_G + 4 * tid);
                tmem_ld32(lane_addr + 0, d);
                tmem_ld_wait();
                const uint4* bsrc = reinterpret_cast<const uint4*>(buf + MW_B + (uint32_t)tid * DVS * 2);
#pragma unroll
                for (int m = 0; m < DVS / 8; ++m) {
                    const uint4 w = bsrc[swz64(tid, m)];
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int j = 8 * m + 2 * p;
                        SB[j] = gamC * SB[j] - d[j] + __uint_as_float(ww[p] << 16);
                        SB[j + 1] = gamC * SB[j + 1] - d[j + 1] + __uint_as_float(ww[p] & 0xFFFF0000u);
                    }
                }
                tmem_ld32(lane_addr + DVS, d);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < DVS; ++j) SM[j] = gamC * SM[j] - d[j];
                mbar_arrive(&bar_free[b]);
                if (it + 1 < nit) write_image();
            }
        }
        __syncthreads();
        if (warp == 5 && lane == 0) {
            for (int j = loads_issued - NBUF < 0 ? 0 : loads_issued - NBUF; j < loads_issued; ++j)
                mbar_wait(&bar_ld[bidx(j)], bpar(j), nullptr);
        }
        if (warp == 4 && lane == 0 && failed && mma_issued > 0) mbar_wait(bar_s, (uint32_t)((mma_issued - 1) & 1), nullptr);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tm, 64);
    }
    if (!consumer) return;
    const size_t st_off = (((size_t)n * H + h) * DK + tid) * DV + (size_t)DVS * jb;
    if (a.trans_out) {
        // row tid, columns [32 jb, 32 jb + 32) of M_g (first half of the output) and B_g
        float* dm = a.trans_out + st_off;
        float* db = a.trans_out + (size_t)a.n_seqs * H * DK * DV + st_off;
#pragma unroll
        for (int j = 0; j < DVS; j += 4) {
            *reinterpret_cast<float4*>(dm + j) = make_float4(SM[j], SM[j + 1], SM[j + 2], SM[j + 3]);
            *reinterpret_cast<float4*>(db + j) = make_float4(SB[j], SB[j + 1], SB[j + 2], SB[j + 3]);
        }
    } else {
        // this segment's slot: B_g as the Bm slice jb, -M_g as the Mlr image (rows tid, K columns
        // [32 jb, 32 jb + 32)), GamC = 0
        uint8_t* slot = a.seg_ws + (((size_t)n * a.segs + g) * H + h) * SLOT_BYTES;
        uint4* dst = reinterpret_cast<uint4*>(slot + SO_B + (size_t)jb * BSL + (size_t)tid * DVS * 2);
#pragma unroll
        for (int m = 0; m < DVS / 8; ++m) dst[swz64(tid, m)] = pack8(SB + 8 * m);
        float nS[DVS];
#pragma unroll
        for (int j = 0; j < DVS; ++j) nS[j] = -SM[j];
        const uint32_t k0 = (uint32_t)(DVS * jb);
        uint8_t* img = slot + SO_M + (size_t)(k0 >> 6) * (DK * 128);
#pragma unroll
        for (int m = 0; m < DVS / 8; ++m)
            *reinterpret_cast<uint4*>(img + sw128_off((uint32_t)tid, (k0 & 63u) + 8u * m)) = pack8(nS + 8 * m);
        if (jb == 0) *reinterpret_cast<float*>(slot + SO_G + 4 * tid) = 0.f;
    }
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

size_t chunk_slot_bytes() { return SLOT_BYTES; }

// Fixed part of the workspace: status word (256 B) + state carry when the
// caller does not ask for the final state.
size_t chunk_fixed_bytes(int n_seqs, int H, bool need_carry) {
    size_t b = 256;
    if (need_carry) b += (size_t)n_seqs * H * DK * DV * sizeof(float);
    return b;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [rows, row_elems] bf16 tensor, box = 64 rows x box_w elements; no swizzle, or the
// 64-byte pattern (16-byte piece m of row r stored at piece m ^ ((r >> 1) & 3), as swz64)
bool make_tile_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems, uint32_t box_w = 128,
                   bool swizzle64 = false) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_elems, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_elems * 2};
    cuuint32_t box[2] = {box_w, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool g_attr_set = false;
int g_num_sms = 0;
// test hook (set_test_tile_drop): consumed by the next chunk-local launch
bool g_drop_tile = false;
unsigned long long g_drop_wait_ns = WAIT_LIMIT_NS;

}  // namespace

bool make_bf16_tile_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems) {
    return make_tile_map(m, base, rows, row_elems);
}

void set_test_tile_drop(unsigned long long wait_ns) {
    g_drop_tile = wait_ns != 0;
    g_drop_wait_ns = wait_ns != 0 ? wait_ns : WAIT_LIMIT_NS;
}

// The chain launch of one pass: SEG as in chain_kernel; gate fused as a 4-CTA cluster.
template <int SEG>
static cudaError_t launch_chain(const ChunkArgs& a, const CUtensorMap& gate_map, const float* norm_w, float eps,
                                bool out_bf16, bool fuse, dim3 gc, cudaStream_t stream) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = gc;
    cfg.blockDim = dim3(CHAIN_THREADS, 1, 1);
    cfg.stream = stream;
    // programmatic serialisation: scheduled while the kernel ahead of it (the chunk-local
    // kernel, or the segment-map walk) still runs; it waits for it before reading slots
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (SEG == 3 || !fuse) {
        cfg.dynamicSmemBytes = ChainLayout<false>::SMEM;
        return out_bf16 ? cudaLaunchKernelEx(&cfg, chain_kernel<true, false, SEG>, a, gate_map, norm_w, eps)
                        : cudaLaunchKernelEx(&cfg, chain_kernel<false, false, SEG>, a, gate_map, norm_w, eps);
    }
    // the four value-column slices of one (sequence, head) form a cluster
    cfg.dynamicSmemBytes = ChainLayout<true>::SMEM;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = CLUSTER;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    if constexpr (SEG == 3) return cudaErrorInvalidValue;  // no outputs, nothing to gate
    else
        return out_bf16 ? cudaLaunchKernelEx(&cfg, chain_kernel<true, true, SEG>, a, gate_map, norm_w, eps)
                        : cudaLaunchKernelEx(&cfg, chain_kernel<false, true, SEG>, a, gate_map, norm_w, eps);
}

template <bool OB, bool G, int SEG>
static cudaError_t set_chain_smem() {
    return cudaFuncSetAttribute(chain_kernel<OB, G, SEG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)ChainLayout<G>::SMEM);
}

// Bytes of the segment slots that follow the chunk slots in segment-parallel mode.
size_t chunk_seg_bytes(int n_seqs, int H, int segs) { return (size_t)n_seqs * segs * H * SLOT_BYTES; }

cudaError_t chunk_fwd_launch(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, void* o, float* final_state, int B, int64_t T, int H,
                             const int32_t* cu, int n_seqs, int64_t max_seqlen, bool in_bf16, bool out_bf16,
                             float scale, const void* gate, const float* norm_w, float eps, float* ckpt,
                             int64_t ckpt_tokens, int segs, int kcp_mode, float* trans_out, void* workspace,
                             size_t ws_bytes, cudaStream_t stream, int* n_passes, bool* gate_fused) {
    cudaError_t err;
    if (!g_attr_set) {
        err = cudaFuncSetAttribute(intra_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, INTRA_SMEM);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(intra_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, INTRA_SMEM);
        if (err != cudaSuccess) return err;
        if ((err = set_chain_smem<true, false, 0>()) != cudaSuccess || (err = set_chain_smem<false, false, 0>()) != cudaSuccess ||
            (err = set_chain_smem<true, true, 0>()) != cudaSuccess || (err = set_chain_smem<false, true, 0>()) != cudaSuccess ||
            (err = set_chain_smem<true, false, 2>()) != cudaSuccess || (err = set_chain_smem<false, false, 2>()) != cudaSuccess ||
            (err = set_chain_smem<true, true, 2>()) != cudaSuccess || (err = set_chain_smem<false, true, 2>()) != cudaSuccess ||
            (err = set_chain_smem<false, false, 3>()) != cudaSuccess ||
            (err = cudaFuncSetAttribute(map_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MW_SMEM)) !=
                cudaSuccess)
            return err;
        int dev = 0;
        if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
        if ((err = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
        g_attr_set = true;
    }
    const int N = cu ? n_seqs : B;
    const int64_t maxlen = cu ? max_seqlen : T;
    const int64_t total_tokens = cu ? T : (int64_t)B * T;
    const int nchunks_max = (int)((maxlen + CH - 1) / CH);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    const bool need_carry = final_state == nullptr;
    // both halves of the cross-device form place the slots after a carry-sized head
    const size_t fixed = chunk_fixed_bytes(N, H, need_carry || kcp_mode != KCP_NONE);
    float* carry = need_carry ? reinterpret_cast<float*>(ws + 256) : final_state;
    const size_t per_wc = (size_t)N * H * SLOT_BYTES;
    const size_t head = (fixed + 1023) & ~(size_t)1023;
    int wc;
    if (segs > 1 || kcp_mode != KCP_NONE) {
        // segment-parallel (segment slots after the chunk slots) and the two halves of
        // the cross-device form: one pass over every chunk
        wc = nchunks_max > 0 ? nchunks_max : 1;
        if (ws_bytes < head + (size_t)wc * per_wc + (segs > 1 ? chunk_seg_bytes(N, H, segs) : 0))
            return cudaErrorInvalidValue;
    } else {
        const size_t wc_fit = ws_bytes > head ? (ws_bytes - head) / per_wc : 0;
        wc = (int)(wc_fit < (size_t)nchunks_max ? wc_fit : (size_t)nchunks_max);
        if (wc < 1) wc = 1;
    }
    ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.init_state = init_state; a.state_io = carry; a.o = o; a.cu = cu;
    a.ws = ws + head;
    a.status = status;
    a.T = T;
    a.H = H; a.n_seqs = N; a.wc = wc; a.scale = scale;
    a.ckpt = ckpt;
    a.ckpt_every = ckpt ? (int)(ckpt_tokens / CH) : 1;
    a.n_ckpt = ckpt ? (int)(maxlen / ckpt_tokens) : 0;
    a.segs = segs > 1 ? segs : 1;
    a.seg_ws = segs > 1 ? a.ws + (size_t)wc * per_wc : nullptr;
    a.trans_out = kcp_mode == KCP_TRANSITION ? trans_out : nullptr;
    a.wait_ns = WAIT_LIMIT_NS;
    a.drop_tile = 0;
    a.wait_first = kcp_mode == KCP_FINISH ? 1 : 0;

    IntraMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (in_bf16 && total_tokens > 0 && kcp_mode != KCP_FINISH) {
        if (!make_tile_map(&maps.la, log_alpha, total_tokens, (int64_t)H * DK) ||
            !make_tile_map(&maps.k, k, total_tokens, (int64_t)H * DK) ||
            !make_tile_map(&maps.q, q, total_tokens, (int64_t)H * DK) ||
            !make_tile_map(&maps.v, v, total_tokens, (int64_t)H * DV))
            return cudaErrorInvalidValue;
    }
    // gate + RMSNorm fused into the chain when the gate is bf16 (its tile
    // arrives by TMA); an fp32 gate is applied by the separate row kernel
    const bool fuse = gate != nullptr && in_bf16;
    CUtensorMap gate_map;
    memset(&gate_map, 0, sizeof(gate_map));
    if (fuse && total_tokens > 0 && !make_tile_map(&gate_map, gate, total_tokens, (int64_t)H * DV, DVS, true))
        return cudaErrorInvalidValue;
    if (gate_fused) *gate_fused = fuse;

    // the finishing half reuses the slots (and the status word) of its transition half
    if (kcp_mode != KCP_FINISH && (err = cudaMemsetAsync(status, 0, 4, stream)) != cudaSuccess) return err;
    if (cu && kcp_mode != KCP_FINISH) {
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
        if (nchunks_max > 0 && kcp_mode != KCP_FINISH) {
            const int64_t n_items = (int64_t)N * wc * H;
            const unsigned grid = (unsigned)(n_items < g_num_sms ? n_items : g_num_sms);
            prof_begin(PROF_INTRA, stream);
            if (g_drop_tile && in_bf16) {  // the test hook applies to one launch
                a.drop_tile = 1;
                a.wait_ns = g_drop_wait_ns;
                g_drop_tile = false;
            }
            if (in_bf16) intra_kernel<true><<<grid, INTRA_THREADS, INTRA_SMEM, stream>>>(a, maps, n_items);
            else intra_kernel<false><<<grid, INTRA_THREADS, INTRA_SMEM, stream>>>(a, maps, n_items);
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
            prof_end(PROF_INTRA, stream);
            a.drop_tile = 0;
            a.wait_ns = WAIT_LIMIT_NS;
        }
        prof_begin(PROF_CHAIN, stream);
        if (o == nullptr && kcp_mode == KCP_NONE && a.segs == 1) {
            // states only (checkpoints, final state): the backward pass's recomputation
            err = launch_chain<3>(a, gate_map, norm_w, eps, false, false, dim3(NSL, H, N), stream);
        } else if (kcp_mode == KCP_TRANSITION) {
            // M_g and B_g of the whole local sequence (one segment), fp32, no outputs
            map_walk_kernel<<<dim3(NSL, H, N), CHAIN_THREADS, MW_SMEM, stream>>>(a);
            err = cudaGetLastError();
        } else if (a.segs == 1) {
            err = launch_chain<0>(a, gate_map, norm_w, eps, out_bf16, fuse, dim3(NSL, H, N), stream);
        } else {
            // segment transitions (no outputs, no gate), then the segments with outputs
            ChunkArgs at = a;
            at.ckpt = nullptr;
            map_walk_kernel<<<dim3(NSL, H, N * a.segs), CHAIN_THREADS, MW_SMEM, stream>>>(at);
            err = cudaGetLastError();
            if (err == cudaSuccess)
                err = launch_chain<2>(a, gate_map, norm_w, eps, out_bf16, fuse, dim3(NSL, H, N * a.segs), stream);
        }
        if (err != cudaSuccess) return err;
        prof_end(PROF_CHAIN, stream);
        ++passes;
    }
    if (n_passes) *n_passes = passes;
    return cudaSuccess;
}

}  // namespace kda
