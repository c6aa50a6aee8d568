// kda_api.cu -- the extern "C" boundary of libkda (declared in include/kda.h).
// Host-side argument checks happen before any launch; every entry point is
// asynchronous on the caller's stream except kda_query_status.
#include <cuda_runtime.h>
#include <stdint.h>

#include <string.h>

#include <vector>

#include "../../include/kda.h"
#include "kda_launch.h"
#include "kda_profile.h"


namespace kda {
namespace {
struct ProfRec {
    int kind;
    cudaEvent_t start, stop;
};
bool g_prof_on = false;
std::vector<ProfRec> g_prof_open;     // begun, not yet ended (at most one per kind)
std::vector<ProfRec> g_prof_done;     // waiting to be read
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
}  // namespace

bool prof_enabled() { return g_prof_on; }

void prof_begin(int kind, cudaStream_t stream) {
    if (!g_prof_on) return;
    ProfRec r{kind, pool_event(), pool_event()};
    cudaEventRecord(r.start, stream);
    g_prof_open.push_back(r);
}

void prof_end(int kind, cudaStream_t stream) {
    if (!g_prof_on) return;
    for (size_t i = g_prof_open.size(); i-- > 0;) {
        if (g_prof_open[i].kind == kind) {
            cudaEventRecord(g_prof_open[i].stop, stream);
            g_prof_done.push_back(g_prof_open[i]);
            g_prof_open.erase(g_prof_open.begin() + (long)i);
            return;
        }
    }
}
}  // namespace kda

namespace {

constexpr int kSupportedD = 128;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(int d) { return d == KDA_F32 || d == KDA_BF16; }

int num_sms_cached() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    return sms;
}

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null pointer, bad size or bad dtype";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: only dk = dv = 128 is implemented";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: pointers must be 16-byte aligned";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or kernel launch failed";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device-side wait gave up";
        case KDA_ERR_DEVICE_ARG: return "KDA_ERR_DEVICE_ARG: cu_seqlens inconsistent with T or max_seqlen";
        default: return "KDA_ERR_UNKNOWN";
    }
}

int kda_version(void) { return 100; }

kda_status kda_chunk_fwd_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen,
                                        size_t* bytes_min, size_t* bytes_full) {
    if (T < 0 || H <= 0 || n_seqs < 0 || max_seqlen < 0 || (!bytes_min && !bytes_full)) return KDA_ERR_INVALID_ARG;
    if (dk != kSupportedD || dv != kSupportedD) return KDA_ERR_UNSUPPORTED;
    // the carry is only needed when final_state is NULL; report the size that
    // covers both cases
    const size_t fixed = kda::chunk_fixed_bytes(n_seqs, H, true);
    const size_t per_wc = (size_t)n_seqs * H * kda::chunk_slot_bytes();
    const int64_t nchunks = (max_seqlen + 63) / 64;
    const size_t head = (fixed + 1023) & ~(size_t)1023;
    if (bytes_min) *bytes_min = head + per_wc + 1024;
    if (bytes_full) *bytes_full = head + per_wc * (size_t)(nchunks > 0 ? nchunks : 1) + 1024;
    return KDA_OK;
}

kda_status kda_chunk_fwd_segmented_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen,
                                                  int segments, size_t* bytes) {
    if (segments < 1 || !bytes) return KDA_ERR_INVALID_ARG;
    size_t full = 0;
    const kda_status st = kda_chunk_fwd_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, nullptr, &full);
    if (st != KDA_OK) return st;
    *bytes = full + (segments > 1 ? kda::chunk_seg_bytes(n_seqs, H, segments) : 0);
    return KDA_OK;
}

static kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const void* log_alpha,
                                 const void* beta, const float* init_state, void* o, float* final_state, int B,
                                 int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, int n_seqs,
                                 int64_t max_seqlen, kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                                 const void* gate, const float* norm_weight, float eps, float* checkpoints,
                                 int64_t ckpt_tokens, int segments, void* workspace, size_t workspace_bytes,
                                 void* stream, int kcp_mode = kda::KCP_NONE, float* transition = nullptr) {
    // the finishing half of the cross-device form reads no token inputs, the
    // transition half writes no outputs; with no tokens at all (an empty segment
    // of a sequence split over devices) the token buffers may be NULL
    const bool has_tokens = B > 0 && T > 0;
    if (has_tokens && kcp_mode != kda::KCP_FINISH && (!q || !k || !v || !log_alpha || !beta))
        return KDA_ERR_INVALID_ARG;
    if (has_tokens && kcp_mode != kda::KCP_TRANSITION && !o) return KDA_ERR_INVALID_ARG;
    if (kcp_mode == kda::KCP_TRANSITION && !transition) return KDA_ERR_INVALID_ARG;
    if (B <= 0 || T < 0 || H <= 0 || !dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_INVALID_ARG;
    if (dk != kSupportedD || dv != kSupportedD) return KDA_ERR_UNSUPPORTED;
    if (H > 65535 || (cu_seqlens ? n_seqs : B) > 65535) return KDA_ERR_UNSUPPORTED;  // grid y / z extents
    if (cu_seqlens) {
        if (B != 1 || n_seqs <= 0 || max_seqlen < 0 || max_seqlen > T) return KDA_ERR_INVALID_ARG;
        if (T > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    } else {
        n_seqs = B;
        max_seqlen = T;
    }
    if ((int64_t)B * T * H * 128 / 128 != (int64_t)B * T * H) return KDA_ERR_INVALID_ARG;
    if (eps < 0.f) return KDA_ERR_INVALID_ARG;
    if (checkpoints && (ckpt_tokens <= 0 || ckpt_tokens % 64 != 0)) return KDA_ERR_INVALID_ARG;
    if (segments < 1) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, gate, norm_weight, workspace,
                          checkpoints, transition};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if (!workspace) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
    size_t need_min = 0;
    const int64_t tot = T * (cu_seqlens ? 1 : B);
    const kda_status wst =
        segments > 1 ? kda_chunk_fwd_segmented_workspace_size(tot, H, dk, dv, n_seqs, max_seqlen, segments, &need_min)
        : kcp_mode != kda::KCP_NONE
            ? kda_chunk_fwd_workspace_size(tot, H, dk, dv, n_seqs, max_seqlen, nullptr, &need_min)
            : kda_chunk_fwd_workspace_size(tot, H, dk, dv, n_seqs, max_seqlen, &need_min, nullptr);
    if (wst != KDA_OK) return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < need_min) return KDA_ERR_WORKSPACE;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool in_bf16 = in_dtype == KDA_BF16, out_bf16 = out_dtype == KDA_BF16;
    bool fused = false;
    cudaError_t e = kda::chunk_fwd_launch(q, k, v, log_alpha, beta, init_state, o, final_state, B, T, H, cu_seqlens,
                                          n_seqs, max_seqlen, in_bf16, out_bf16, scale, gate, norm_weight, eps,
                                          checkpoints, ckpt_tokens, segments, kcp_mode, transition, workspace,
                                          workspace_bytes, st, nullptr,
                                          &fused);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    if (gate && !fused && kcp_mode != kda::KCP_TRANSITION) {
        const int64_t rows = (int64_t)B * T * H;
        // y overwrites o in place (o already holds out_dtype values)
        kda::prof_begin(kda::PROF_GATE_NORM, st);
        e = kda::launch_gate_norm(o, gate, norm_weight, eps, o, rows, out_bf16, in_bf16, out_bf16, num_sms_cached(),
                                  st);
        kda::prof_end(kda::PROF_GATE_NORM, st);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

kda_status kda_chunk_fwd_ckpt(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* init_state, void* o, float* final_state, int B, int64_t T, int H, int dk,
                              int dv, const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen, kda_dtype in_dtype,
                              kda_dtype out_dtype, float scale, const void* gate, const float* norm_weight, float eps,
                              float* checkpoints, int64_t ckpt_tokens, void* workspace, size_t workspace_bytes,
                              void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, init_state, o, final_state, B, T, H, dk, dv, cu_seqlens, n_seqs,
                          max_seqlen, in_dtype, out_dtype, scale, gate, norm_weight, eps, checkpoints, ckpt_tokens, 1,
                          workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_segmented(const void* q, const void* k, const void* v, const void* log_alpha,
                                   const void* beta, const float* init_state, void* o, float* final_state, int B,
                                   int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, int n_seqs,
                                   int64_t max_seqlen, kda_dtype in_dtype, kda_dtype out_dtype, float scale,
                                   const void* gate, const float* norm_weight, float eps, int segments,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, init_state, o, final_state, B, T, H, dk, dv, cu_seqlens, n_seqs,
                          max_seqlen, in_dtype, out_dtype, scale, gate, norm_weight, eps, nullptr, 0, segments,
                          workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                         const float* init_state, void* o, float* final_state, int B, int64_t T, int H, int dk,
                         int dv, const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen, kda_dtype in_dtype,
                         kda_dtype out_dtype, float scale, const void* gate, const float* norm_weight, float eps,
                         void* workspace, size_t workspace_bytes, void* stream) {
    return kda_chunk_fwd_ckpt(q, k, v, log_alpha, beta, init_state, o, final_state, B, T, H, dk, dv, cu_seqlens, n_seqs,
                              max_seqlen, in_dtype, out_dtype, scale, gate, norm_weight, eps, nullptr, 0, workspace,
                              workspace_bytes, stream);
}

kda_status kda_kcp_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen, size_t* bytes) {
    if (!bytes) return KDA_ERR_INVALID_ARG;
    return kda_chunk_fwd_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, nullptr, bytes);
}

kda_status kda_kcp_transition(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              int B, int64_t T, int H, int dk, int dv, const int32_t* cu_seqlens, int n_seqs,
                              int64_t max_seqlen, kda_dtype in_dtype, float scale, float* transition,
                              void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, nullptr, nullptr, nullptr, B, T, H, dk, dv, cu_seqlens, n_seqs,
                          max_seqlen, in_dtype, in_dtype, scale, nullptr, nullptr, 0.f, nullptr, 0, 1, workspace,
                          workspace_bytes, stream, kda::KCP_TRANSITION, transition);
}

kda_status kda_kcp_compose(const float* transitions, int n_prev, const float* init_state, float* state_in,
                           int n_seqs, int H, int dk, int dv, void* stream) {
    if (!state_in || n_prev < 0 || (n_prev > 0 && !transitions) || n_seqs < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kSupportedD || dv != kSupportedD) return KDA_ERR_UNSUPPORTED;
    if (H > 65535 || n_seqs > 65535) return KDA_ERR_UNSUPPORTED;
    const void* ptrs[] = {transitions, init_state, state_in};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    return from_cuda(kda::launch_kcp_compose(transitions, n_prev, init_state, state_in, n_seqs, H,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

kda_status kda_kcp_finish(const float* state_in, void* o, float* final_state, int B, int64_t T, int H, int dk, int dv,
                          const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen, kda_dtype in_dtype,
                          kda_dtype out_dtype, const void* gate, const float* norm_weight, float eps,
                          void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(nullptr, nullptr, nullptr, nullptr, nullptr, state_in, o, final_state, B, T, H, dk, dv,
                          cu_seqlens, n_seqs, max_seqlen, in_dtype, out_dtype, 1.f, gate, norm_weight, eps, nullptr, 0,
                          1, workspace, workspace_bytes, stream, kda::KCP_FINISH, nullptr);
}

kda_status kda_chunk_bwd_workspace_size(int64_t T, int H, int dk, int dv, int n_seqs, int64_t max_seqlen,
                                       size_t* bytes) {
    if (!bytes) return KDA_ERR_INVALID_ARG;
    size_t full = 0;
    const kda_status st = kda_chunk_fwd_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, nullptr, &full);
    if (st != KDA_OK) return st;
    *bytes = full + kda::chunk_bwd_extra_bytes(n_seqs, H, max_seqlen);
    return KDA_OK;
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                         const float* init_state, const void* d_o, const float* d_final_state, float* dq, float* dk,
                         float* dv, float* dlog_alpha, float* dbeta, float* d_init_state, int B, int64_t T, int H,
                         int dk_dim, int dv_dim, const int32_t* cu_seqlens, int n_seqs, int64_t max_seqlen,
                         kda_dtype in_dtype, float scale, void* workspace, size_t workspace_bytes, void* stream) {
    if (B <= 0 || T < 0 || H <= 0 || !dtype_ok(in_dtype)) return KDA_ERR_INVALID_ARG;
    if (dk_dim != kSupportedD || dv_dim != kSupportedD) return KDA_ERR_UNSUPPORTED;
    if (H > 65535 || (cu_seqlens ? n_seqs : B) > 65535) return KDA_ERR_UNSUPPORTED;
    const bool has_tokens = T > 0;
    if (has_tokens && (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk || !dv || !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1 || n_seqs <= 0 || max_seqlen < 0 || max_seqlen > T) return KDA_ERR_INVALID_ARG;
        if (T > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    } else {
        n_seqs = B;
        max_seqlen = T;
    }
    const void* ptrs[] = {q,  k,  v,  log_alpha, beta,  init_state, d_o,          d_final_state, dq,
                          dk, dv, dlog_alpha, dbeta, d_init_state, cu_seqlens, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if (!workspace) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
    const int64_t tot = T * (cu_seqlens ? 1 : B);
    size_t fwd_full = 0, need = 0;
    if (kda_chunk_fwd_workspace_size(tot, H, dk_dim, dv_dim, n_seqs, max_seqlen, nullptr, &fwd_full) != KDA_OK ||
        kda_chunk_bwd_workspace_size(tot, H, dk_dim, dv_dim, n_seqs, max_seqlen, &need) != KDA_OK)
        return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    const cudaError_t e = kda::chunk_bwd_launch(q, k, v, log_alpha, beta, init_state, d_o, d_final_state, dq, dk, dv,
                                                dlog_alpha, dbeta, d_init_state, B, T, H, cu_seqlens, n_seqs,
                                                max_seqlen, in_dtype == KDA_BF16, scale, workspace, fwd_full,
                                                reinterpret_cast<cudaStream_t>(stream));
    return from_cuda(e);
}

kda_status kda_decode_steps(float* state, const void* q, const void* k, const void* v, const void* log_alpha,
                            const void* beta, void* o, int n_steps, int Bd, int H, int dk, int dv,
                            kda_dtype in_dtype, kda_dtype out_dtype, float scale, const void* gate,
                            const float* norm_weight, float eps, float* step_states, void* stream) {
    if (!state || !q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_INVALID_ARG;
    if (n_steps < 0 || Bd < 0 || H <= 0 || !dtype_ok(in_dtype) || !dtype_ok(out_dtype) || eps < 0.f)
        return KDA_ERR_INVALID_ARG;
    if (dk != kSupportedD || dv != kSupportedD) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)Bd * H > INT32_MAX) return KDA_ERR_UNSUPPORTED;
    const void* ptrs[] = {state, q, k, v, log_alpha, beta, o, gate, norm_weight, step_states};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if (Bd == 0 || n_steps == 0) return KDA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    kda::prof_begin(kda::PROF_DECODE, st);
    const cudaError_t e = kda::launch_decode_step(state, q, k, v, log_alpha, beta, o, Bd, H, in_dtype == KDA_BF16,
                                                  out_dtype == KDA_BF16, scale, gate, norm_weight, eps, n_steps,
                                                  step_states, st);
    kda::prof_end(kda::PROF_DECODE, st);
    return from_cuda(e);
}

kda_status kda_decode_step(float* state, const void* q, const void* k, const void* v, const void* log_alpha,
                           const void* beta, void* o, int Bd, int H, int dk, int dv, kda_dtype in_dtype,
                           kda_dtype out_dtype, float scale, const void* gate, const float* norm_weight, float eps,
                           void* stream) {
    return kda_decode_steps(state, q, k, v, log_alpha, beta, o, 1, Bd, H, dk, dv, in_dtype, out_dtype, scale, gate,
                            norm_weight, eps, nullptr, stream);
}

kda_status kda_gate_norm(const void* o, const void* gate, const float* norm_weight, float eps, void* y, int64_t rows,
                         int dv, kda_dtype in_dtype, kda_dtype out_dtype, void* stream) {
    if (!o || !gate || !y || rows < 0 || !dtype_ok(in_dtype) || !dtype_ok(out_dtype) || eps < 0.f)
        return KDA_ERR_INVALID_ARG;
    if (dv != kSupportedD) return KDA_ERR_UNSUPPORTED;
    if (y == o && in_dtype != out_dtype) return KDA_ERR_INVALID_ARG;  // in place needs equal element sizes
    const void* ptrs[] = {o, gate, norm_weight, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    kda::prof_begin(kda::PROF_GATE_NORM, st);
    const cudaError_t e = kda::launch_gate_norm(o, gate, norm_weight, eps, y, rows, in_dtype == KDA_BF16,
                                                in_dtype == KDA_BF16, out_dtype == KDA_BF16, num_sms_cached(), st);
    kda::prof_end(kda::PROF_GATE_NORM, st);
    return from_cuda(e);
}

kda_status kda_profile_enable(int on) {
    kda::g_prof_on = on != 0;
    return KDA_OK;
}

kda_status kda_profile_read(kda_kernel_time* out, int max_entries, int* n_entries) {
    static const char* names[kda::PROF_KINDS] = {"intra",      "chain",    "gate_norm",
                                                 "decode",     "check_cu", "kcp_compose",
                                                 "chain_bwd",  "intra_bwd"};
    int launches[kda::PROF_KINDS] = {0};
    double ms[kda::PROF_KINDS] = {0};
    kda_status st = KDA_OK;
    for (auto& r : kda::g_prof_done) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            st = KDA_ERR_CUDA;
        launches[r.kind] += 1;
        ms[r.kind] += t;
        kda::g_event_pool.push_back(r.start);
        kda::g_event_pool.push_back(r.stop);
    }
    kda::g_prof_done.clear();
    int n = 0;
    for (int k = 0; k < kda::PROF_KINDS; ++k) {
        if (launches[k] == 0) continue;
        if (out && n < max_entries) {
            memset(out[n].name, 0, sizeof(out[n].name));
            strncpy(out[n].name, names[k], sizeof(out[n].name) - 1);
            out[n].launches = launches[k];
            out[n].ms = ms[k];
        }
        ++n;
    }
    if (n_entries) *n_entries = n;
    return st;
}

kda_status kda_test_drop_tile_load(unsigned long long wait_limit_ns) {
    if (wait_limit_ns != 0 && (wait_limit_ns < 1000ull || wait_limit_ns > 1000000000ull)) return KDA_ERR_INVALID_ARG;
    kda::set_test_tile_drop(wait_limit_ns);
    return KDA_OK;
}

kda_status kda_query_status(void* workspace, void* stream) {
    if (!workspace) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    if (word & 1u) return KDA_ERR_TIMEOUT;
    if (word & 2u) return KDA_ERR_DEVICE_ARG;
    return KDA_OK;
}

}  // extern "C"
