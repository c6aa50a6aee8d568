// kda_decode.cu -- recurrent decode step and the per-head RMSNorm + sigmoid
// output gate.  Both are HBM-bound: decode streams each head's fp32 state
// once in and once out; gate-norm streams o and g once.
//
// Recurrent form (K3 article summaries, xhh.club tag page, items "KDA
// recurrence form" and "chunkwise parallel algorithm": decode uses the
// recurrence).  Per head, with S' = Diag(alpha) S:
//     u = beta (v - S'^T k);   S_new = S' + k u^T;   o = scale * S_new^T q
// and o = scale * (S'^T q + (k . q) u), so both dot products over the key
// channels come from ONE pass over S' and the state is read and written once.
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {

// One CTA = one (sequence, head) state [128 x 128] fp32 = 64 KiB, carried
// through n_steps consecutive tokens; the state is read once and written once
// for all of them, and optionally also after every step.  The launcher uses it
// for single steps with the output gate fused (GATE: the per-head RMSNorm needs
// all 128 value columns of the head in one CTA); ungated steps and several steps
// per call go to decode_multi_kernel below.
// 256 threads = 8 warps; warp w owns value columns [16w, 16w + 16).
// Lane l: row phase r0 = l / 4 (0..7) and column quad cq = l % 4, so one warp
// load instruction covers 8 rows x 64 contiguous bytes.  Thread holds rows
// r0 + 8i (i = 0..15) x 4 columns = 64 fp32 registers.
// Token tensors are step-major: element (step t, sequence-head bh, channel c)
// at (t * BH + bh) * 128 + c (beta: t * BH + bh).
template <bool IN_BF16, bool OUT_BF16, bool GATE>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(float* __restrict__ state, const void* __restrict__ q, const void* __restrict__ k,
                   const void* __restrict__ v, const void* __restrict__ log_alpha,
                   const void* __restrict__ beta, void* __restrict__ o, const void* __restrict__ gate,
                   const float* __restrict__ norm_w, float scale, float eps, int n_steps,
                   float* __restrict__ step_states) {
    constexpr int D = 128;
    const int bh = blockIdx.x;  // sequence * H + head
    const size_t BH = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = lane >> 2, cq = lane & 3;
    const int col = warp * 16 + cq * 4;

    // per-step token vectors, double-buffered by step parity (the buffer of step
    // t is rewritten at step t + 2, after the barrier of step t + 1)
    __shared__ float s_k[2][D], s_q[2][D], s_alpha[2][D];
    __shared__ float s_ss[2][8];

    float* S = state + (size_t)bh * D * D;
    float4 st[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        st[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(r0 + 8 * i) * D + col));

    // this step's token values, loaded one step ahead into registers
    float nk = 0.f, nq = 0.f, nla = 0.f, nb, nv[4], ng[4];
    auto load_step = [&](int t) {
        const size_t tb = (size_t)t * BH + bh;
        if (tid < D) {
            const size_t idx = tb * D + tid;
            nk = ld_in<IN_BF16>(k, idx);
            nq = ld_in<IN_BF16>(q, idx);
            nla = ld_in<IN_BF16>(log_alpha, idx);
        }
        nb = ld_in<IN_BF16>(beta, tb);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            nv[c] = ld_in<IN_BF16>(v, tb * D + col + c);
            if constexpr (GATE) ng[c] = ld_in<IN_BF16>(gate, tb * D + col + c);
        }
    };
    load_step(0);

    for (int t = 0; t < n_steps; ++t) {
        const int pb = t & 1;
        const size_t tb = (size_t)t * BH + bh;  // token row of this step
        if (tid < D) {
            s_k[pb][tid] = nk;
            s_q[pb][tid] = nq;
            s_alpha[pb][tid] = __expf(fmaxf(nla, LOG_ALPHA_FLOOR));
        }
        const float b = nb;
        float vv[4], gg4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            vv[c] = nv[c];
            gg4[c] = GATE ? ng[c] : 0.f;
        }
        if (t + 1 < n_steps) load_step(t + 1);  // in flight during this step
        __syncthreads();
        const float* sk_ = s_k[pb];
        const float* sq_ = s_q[pb];
        const float* sa_ = s_alpha[pb];

        // k . q (every warp computes it; 4 products per lane + butterfly)
        float kq = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) kq += sk_[lane + 32 * m] * sq_[lane + 32 * m];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, m);

        // decay rows, partial S'^T k and S'^T q over this thread's 16 rows
        float sk[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = r0 + 8 * i;
            const float a = sa_[r], kr = sk_[r], qr = sq_[r];
            st[i].x *= a; st[i].y *= a; st[i].z *= a; st[i].w *= a;
            sk[0] += st[i].x * kr; sk[1] += st[i].y * kr; sk[2] += st[i].z * kr; sk[3] += st[i].w * kr;
            sq[0] += st[i].x * qr; sq[1] += st[i].y * qr; sq[2] += st[i].z * qr; sq[3] += st[i].w * qr;
        }
        // reduce over the 8 row phases (lanes that share cq)
#pragma unroll
        for (int m = 4; m <= 16; m <<= 1) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                sk[c] += __shfl_xor_sync(0xffffffffu, sk[c], m);
                sq[c] += __shfl_xor_sync(0xffffffffu, sq[c], m);
            }
        }
        float u[4], oc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            u[c] = b * (vv[c] - sk[c]);
            oc[c] = scale * (sq[c] + kq * u[c]);
        }
        // S_new = S' + k u^T; this step's state when the caller keeps them, and the
        // carried state written back once, at the last step
        float* SS = step_states ? step_states + tb * D * D : nullptr;
        const bool last = t + 1 == n_steps;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float kr = sk_[r0 + 8 * i];
            st[i].x += kr * u[0]; st[i].y += kr * u[1]; st[i].z += kr * u[2]; st[i].w += kr * u[3];
            if (SS) __stcs(reinterpret_cast<float4*>(SS + (size_t)(r0 + 8 * i) * D + col), st[i]);
            if (last) __stcs(reinterpret_cast<float4*>(S + (size_t)(r0 + 8 * i) * D + col), st[i]);
        }

        if constexpr (GATE) {
            // per-head RMSNorm over the 128 value channels, then weight and gate
            float ss = oc[0] * oc[0] + oc[1] * oc[1] + oc[2] * oc[2] + oc[3] * oc[3];
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            if (lane == 0) s_ss[pb][warp] = ss;
            __syncthreads();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) tot += s_ss[pb][w];
            const float inv = rsqrtf(tot * (1.0f / D) + eps);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float wc = norm_w ? __ldg(norm_w + col + c) : 1.0f;
                oc[c] = oc[c] * inv * wc * __fdividef(1.0f, 1.0f + __expf(-gg4[c]));
            }
        }
        if (r0 == 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) st_out<OUT_BF16>(o, tb * D + col + c, oc[c]);
        }
    }
}

// Ungated steps, one or several per call: the head's columns are split over two CTAs of
// 128 threads (the columns evolve independently given the token's k, q, alpha, beta),
// so twice as many, half-size CTAs are in flight per SM and the loads, steps and stores
// of different CTAs overlap when a call runs several steps.  Warp w of slice sl owns
// columns [64 sl + 16 w, +16); lane l: row block rb = l / 8 (rows 32 rb .. 32 rb + 31,
// contiguous) and column pair cp = l % 8 (columns 2 cp, 2 cp + 1 of the warp's 16): a
// thread holds 32 rows x 2 columns (64 fp32 registers), reads the rows' decay, k and q
// four at a time (16-byte shared loads), and the column sums need one 4-lane reduction.
// Per step and column: S' = alpha o S;  u = beta (v - S'^T k);  o = scale (S'^T q + (k.q) u);
// S = S' + k u^T, the same arithmetic whatever the number of steps per call.
// The token rows of up to DECODE_BLOCK steps (k, q, log_alpha and the CTA's half of v)
// arrive together by asynchronous copies into shared memory, the first block's in the
// shadow of the state load, and are converted once per block into fp32 per-row vectors
// (k, q, alpha = e^l) and v columns: the steps of a block then wait for no global load
// (a step is shorter than the latency of one under a full HBM load) and for no barrier,
// so the warps of a CTA run through them independently.
constexpr int DECODE_BLOCK = 8;

KDA_DEV void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
KDA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
KDA_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(128, 4)
decode_multi_kernel(float* __restrict__ state, const void* __restrict__ q, const void* __restrict__ k,
                    const void* __restrict__ v, const void* __restrict__ log_alpha, const void* __restrict__ beta,
                    void* __restrict__ o, float scale, int n_steps, float* __restrict__ step_states) {
    constexpr int D = 128;
    const int bh = blockIdx.x >> 1, sl = blockIdx.x & 1;  // (sequence * H + head, column half)
    const size_t BH = gridDim.x >> 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rb = lane >> 3, cp = lane & 7;
    const int col = 64 * sl + 16 * warp + 2 * cp;
    const int row0 = 32 * rb;
    // per-row token values, rows of block rb at offset 36 rb (4 floats of padding per block):
    // the four row blocks a warp reads at once fall into different banks
    constexpr int DP = D + 12;
    __shared__ __align__(16) float s_k[DECODE_BLOCK][DP], s_q[DECODE_BLOCK][DP], s_alpha[DECODE_BLOCK][DP];
    __shared__ float s_v[DECODE_BLOCK][64];
    const int pr = tid + 4 * (tid >> 5);   // padded slot of row tid
    const int prow0 = row0 + 4 * rb;       // padded slot of this thread's first row
    // a block of steps' raw token rows: per step [k | q | log_alpha] rows of 128 elements and
    // this CTA's 64 elements of v, then beta per step
    constexpr int ES = IN_BF16 ? 2 : 4;
    constexpr int ROWB = D * ES, VB = 64 * ES, STEPB = 3 * ROWB + VB;
    __shared__ __align__(16) uint8_t s_tok[DECODE_BLOCK * STEPB];
    __shared__ float s_beta[DECODE_BLOCK];
    auto tok = [&](int s_, int part, int e) -> float {  // element e of part (0 k, 1 q, 2 log_alpha, 3 v)
        const uint8_t* p = s_tok + s_ * STEPB + part * ROWB + e * ES;
        if constexpr (IN_BF16) return __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(p) << 16);
        else return *reinterpret_cast<const float*>(p);
    };
    // copies of steps [t0, t0 + nb): 16-byte pieces, CHUNK_ROW per row, CHUNK_V for v
    auto fetch_block = [&](int t0) {
        const int nb = n_steps - t0 < DECODE_BLOCK ? n_steps - t0 : DECODE_BLOCK;
        constexpr int CR = ROWB / 16, CV = VB / 16, CS = 3 * CR + CV;
        for (int ci = tid; ci < nb * CS; ci += 128) {
            const int s_ = ci / CS, r = ci - s_ * CS;
            const size_t tb = (size_t)(t0 + s_) * BH + bh;
            const uint8_t* src;
            if (r < 3 * CR) {
                const int part = r / CR;
                const void* base = part == 0 ? k : (part == 1 ? q : log_alpha);
                src = reinterpret_cast<const uint8_t*>(base) + tb * ROWB + (size_t)(r - part * CR) * 16;
            } else {
                src = reinterpret_cast<const uint8_t*>(v) + tb * ROWB + (size_t)sl * VB + (size_t)(r - 3 * CR) * 16;
            }
            cp_async16(s_tok + s_ * STEPB + r * 16, src);
        }
        cp_async_commit();
        // beta of step t0 + tid: kept in a register until the block's wait
        return tid < nb ? ld_in<IN_BF16>(beta, (size_t)(t0 + tid) * BH + bh) : 0.f;
    };
    float beta_next = fetch_block(0);  // in flight with the state load

    float* S = state + (size_t)bh * D * D;
    float2 st[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) st[i] = __ldcs(reinterpret_cast<const float2*>(S + (size_t)(row0 + i) * D + col));

    const int vc = col - 64 * sl;  // this thread's v columns within the CTA's half
    for (int t = 0; t < n_steps; ++t) {
        const size_t tb = (size_t)t * BH + bh;
        const int s_ = t % DECODE_BLOCK;
        if (s_ == 0) {
            // s_tok was last read by the previous block's conversion, which every thread
            // finished before that block's second barrier
            if (t > 0) beta_next = fetch_block(t);
            cp_async_wait_all();
            __syncthreads();  // the copies have landed; every thread is done with the last block's vectors
            const int nb = n_steps - t < DECODE_BLOCK ? n_steps - t : DECODE_BLOCK;
            for (int j = 0; j < nb; ++j) {
                s_k[j][pr] = tok(j, 0, tid);
                s_q[j][pr] = tok(j, 1, tid);
                s_alpha[j][pr] = __expf(fmaxf(tok(j, 2, tid), LOG_ALPHA_FLOOR));
                if (tid < 64) s_v[j][tid] = tok(j, 3, tid);
            }
            if (tid < DECODE_BLOCK) s_beta[tid] = beta_next;
            __syncthreads();
        }
        const float b = s_beta[s_], v0 = s_v[s_][vc], v1 = s_v[s_][vc + 1];
        const float* sk_ = s_k[s_];
        const float* sq_ = s_q[s_];
        const float* sa_ = s_alpha[s_];

        float kq = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) kq += sk_[lane + 36 * m] * sq_[lane + 36 * m];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, m);

        // decay the rows, partial S'^T k and S'^T q over this thread's 32 rows; the two
        // columns of a row go through the paired fp32 instructions (each half rounds as
        // the scalar one would)
        // (two partial sums per dot product: even and odd row groups, half the dependent chain)
        float2 skv = make_float2(0.f, 0.f), sqv = make_float2(0.f, 0.f);
        float2 skw = make_float2(0.f, 0.f), sqw = make_float2(0.f, 0.f);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
            const float4 a4 = *reinterpret_cast<const float4*>(sa_ + prow0 + 4 * i4);
            const float4 k4 = *reinterpret_cast<const float4*>(sk_ + prow0 + 4 * i4);
            const float4 q4 = *reinterpret_cast<const float4*>(sq_ + prow0 + 4 * i4);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w},
                        qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2& x = st[4 * i4 + e];
                x = __fmul2_rn(x, make_float2(av[e], av[e]));
                if (e & 1) {
                    skw = __ffma2_rn(x, make_float2(kv[e], kv[e]), skw);
                    sqw = __ffma2_rn(x, make_float2(qv[e], qv[e]), sqw);
                } else {
                    skv = __ffma2_rn(x, make_float2(kv[e], kv[e]), skv);
                    sqv = __ffma2_rn(x, make_float2(qv[e], qv[e]), sqv);
                }
            }
        }
        float sk0 = skv.x + skw.x, sk1 = skv.y + skw.y, sq0 = sqv.x + sqw.x, sq1 = sqv.y + sqw.y;
        // reduce over the 4 row blocks (lanes that share cp)
#pragma unroll
        for (int m = 8; m <= 16; m <<= 1) {
            sk0 += __shfl_xor_sync(0xffffffffu, sk0, m);
            sk1 += __shfl_xor_sync(0xffffffffu, sk1, m);
            sq0 += __shfl_xor_sync(0xffffffffu, sq0, m);
            sq1 += __shfl_xor_sync(0xffffffffu, sq1, m);
        }
        const float u0 = b * (v0 - sk0), u1 = b * (v1 - sk1);
        const float o0 = scale * (sq0 + kq * u0), o1 = scale * (sq1 + kq * u1);
        const float2 u2 = make_float2(u0, u1);
        // S = S' + k u^T; this step's state when the caller keeps them, and the carried
        // state written back once, at the last step
        float* SS = step_states ? step_states + tb * D * D : nullptr;
        const bool last = t + 1 == n_steps;
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
            const float4 k4 = *reinterpret_cast<const float4*>(sk_ + prow0 + 4 * i4);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) st[4 * i4 + e] = __ffma2_rn(make_float2(kv[e], kv[e]), u2, st[4 * i4 + e]);
        }
        if (SS || last) {
            float* dst = (SS ? SS : S) + (size_t)row0 * D + col;
#pragma unroll
            for (int i = 0; i < 32; ++i) __stcs(reinterpret_cast<float2*>(dst + (size_t)i * D), st[i]);
            if (SS && last) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    __stcs(reinterpret_cast<float2*>(S + (size_t)(row0 + i) * D + col), st[i]);
            }
        }
        if (rb == 0) {
            if constexpr (OUT_BF16) {
                *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(o) + tb * D + col) = pack_bf16x2(o0, o1);
            } else {
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(o) + tb * D + col) = make_float2(o0, o1);
            }
        }
    }
}

// y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) over rows of dv = 128.
// Half a warp per row (8 consecutive channels = 16 bytes of bf16 per lane),
// two rows per warp, grid-stride over row pairs (warp-uniform trip count).  In place (y == o) is safe:
// each half-warp reads its whole row before it writes it.
template <bool BF>
KDA_DEV void load8(const void* base, size_t idx, float* v) {
    if constexpr (BF) {
        const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + idx);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            v[2 * p] = __uint_as_float(ww[p] << 16);
            v[2 * p + 1] = __uint_as_float(ww[p] & 0xFFFF0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
        const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

template <bool O_BF16, bool G_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(256)
gate_norm_kernel(const void* o, const void* __restrict__ g, const float* __restrict__ norm_w, float eps,
                 void* y, int64_t rows) {
    constexpr int D = 128;
    const int lane = threadIdx.x & 31, sub = lane & 15;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    float w8[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) w8[c] = norm_w ? __ldg(norm_w + sub * 8 + c) : 1.0f;
    // the loop runs over row pairs so that every lane of a warp takes the same
    // number of iterations (the shuffles below use the full mask)
    for (int64_t pair = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); 2 * pair < rows;
         pair += warps_total) {
        const int64_t row = 2 * pair + (lane >> 4);
        const bool valid = row < rows;
        const size_t base = (size_t)row * D + sub * 8;
        float ov[8], gv[8];
        if (valid) {
            load8<O_BF16>(o, base, ov);
            load8<G_BF16>(g, base, gv);
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) ov[c] = gv[c] = 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) ss += ov[c] * ov[c];
#pragma unroll
        for (int m = 8; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float inv = rsqrtf(ss * (1.0f / D) + eps);
        float yv[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) yv[c] = ov[c] * inv * w8[c] * __fdividef(1.0f, 1.0f + __expf(-gv[c]));
        if (!valid) continue;
        if constexpr (OUT_BF16) {
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + base) =
                make_uint4(pack_bf16x2(yv[0], yv[1]), pack_bf16x2(yv[2], yv[3]), pack_bf16x2(yv[4], yv[5]),
                           pack_bf16x2(yv[6], yv[7]));
        } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + base);
            dst[0] = make_float4(yv[0], yv[1], yv[2], yv[3]);
            dst[1] = make_float4(yv[4], yv[5], yv[6], yv[7]);
        }
    }
}

// ------------------------------------------------------------ launchers --

cudaError_t launch_decode_step(float* state, const void* q, const void* k, const void* v,
                               const void* log_alpha, const void* beta, void* o, int Bd, int H,
                               bool in_bf16, bool out_bf16, float scale, const void* gate,
                               const float* norm_w, float eps, int n_steps, float* step_states,
                               cudaStream_t stream) {
    const bool g = gate != nullptr;
    if (g && n_steps == 1) {  // one step with the gate fused: one CTA per (sequence, head)
        const dim3 grid((unsigned)((int64_t)Bd * H)), block(256);
#define KDA_DEC(IB, OB)                                                                                    \
    decode_step_kernel<IB, OB, true><<<grid, block, 0, stream>>>(state, q, k, v, log_alpha, beta, o, gate, \
                                                                 norm_w, scale, eps, n_steps, step_states)
        if (in_bf16) { if (out_bf16) KDA_DEC(true, true); else KDA_DEC(true, false); }
        else         { if (out_bf16) KDA_DEC(false, true); else KDA_DEC(false, false); }
#undef KDA_DEC
        return cudaGetLastError();
    }
    // two half-head CTAs per (sequence, head); with a gate, the per-head RMSNorm and gate
    // then run over the n_steps output rows in place
    const dim3 grid((unsigned)((int64_t)Bd * H * 2)), block(128);
#define KDA_DECM(IB, OB)                                                                               \
    decode_multi_kernel<IB, OB><<<grid, block, 0, stream>>>(state, q, k, v, log_alpha, beta, o, scale, \
                                                            n_steps, step_states)
    if (in_bf16) { if (out_bf16) KDA_DECM(true, true); else KDA_DECM(true, false); }
    else         { if (out_bf16) KDA_DECM(false, true); else KDA_DECM(false, false); }
#undef KDA_DECM
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || !g) return err;
    int dev = 0, sms = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    return launch_gate_norm(o, gate, norm_w, eps, o, (int64_t)n_steps * Bd * H, out_bf16, in_bf16, out_bf16, sms,
                            stream);
}

cudaError_t launch_gate_norm(const void* o, const void* g, const float* norm_w, float eps, void* y,
                             int64_t rows, bool o_bf16, bool g_bf16, bool out_bf16, int num_sms,
                             cudaStream_t stream) {
    const int64_t blocks_needed = (rows + 15) / 16;  // 16 rows per 256-thread block
    const int64_t cap = (int64_t)num_sms * 8;
    const dim3 grid((unsigned)(blocks_needed < cap ? blocks_needed : cap)), block(256);
    if (rows == 0) return cudaSuccess;
#define KDA_GN(OB, GB, YB) gate_norm_kernel<OB, GB, YB><<<grid, block, 0, stream>>>(o, g, norm_w, eps, y, rows)
    if (o_bf16) {
        if (g_bf16) { if (out_bf16) KDA_GN(true, true, true); else KDA_GN(true, true, false); }
        else        { if (out_bf16) KDA_GN(true, false, true); else KDA_GN(true, false, false); }
    } else {
        if (g_bf16) { if (out_bf16) KDA_GN(false, true, true); else KDA_GN(false, true, false); }
        else        { if (out_bf16) KDA_GN(false, false, true); else KDA_GN(false, false, false); }
    }
#undef KDA_GN
    return cudaGetLastError();
}

}  // namespace kda
