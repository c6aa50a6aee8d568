// kda_launch.h -- host-side launchers behind the C ABI (internal to libkda).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

// The two halves of the cross-device (context-parallel) prefill of a sequence
// split over devices.  KCP_TRANSITION runs the chunk-local kernel over every
// chunk, keeps its slots in the workspace and writes the segment's affine state
// map (M, B) in fp32; KCP_FINISH walks the kept slots from the initial state
// that the maps of the earlier segments produced, with outputs.
enum KcpMode { KCP_NONE = 0, KCP_TRANSITION = 1, KCP_FINISH = 2 };

cudaError_t launch_decode_step(float* state, const void* q, const void* k, const void* v, const void* log_alpha,
                               const void* beta, void* o, int Bd, int H, bool in_bf16, bool out_bf16, float scale,
                               const void* gate, const float* norm_w, float eps, int n_steps, float* step_states,
                               cudaStream_t stream);
cudaError_t launch_gate_norm(const void* o, const void* g, const float* norm_w, float eps, void* y, int64_t rows,
                             bool o_bf16, bool g_bf16, bool out_bf16, int num_sms, cudaStream_t stream);
size_t chunk_slot_bytes();
size_t chunk_fixed_bytes(int n_seqs, int H, bool need_carry);
size_t chunk_seg_bytes(int n_seqs, int H, int segs);
cudaError_t chunk_fwd_launch(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, void* o, float* final_state, int B, int64_t T, int H,
                             const int32_t* cu, int n_seqs, int64_t max_seqlen, bool in_bf16, bool out_bf16,
                             float scale, const void* gate, const float* norm_w, float eps, float* ckpt,
                             int64_t ckpt_tokens, int segs, int kcp_mode, float* trans_out, void* workspace,
                             size_t ws_bytes, cudaStream_t stream, int* n_passes, bool* gate_fused);
// 2-D tensor map of a [rows, row_elems] bf16 tensor with a box of 64 rows x 128
// elements, no swizzle (the chunk-local kernels' tile loads).  False on failure.
bool make_bf16_tile_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_elems);

// Test hook: the next chunk-local launch with bf16 inputs has CTA 0 skip one of
// its first item's four tile loads and give up waiting after wait_ns (0 cancels).
void set_test_tile_drop(unsigned long long wait_ns);

// state_in = fold of maps 0 .. n_prev-1 of `trans` over init_state (zero when null)
cudaError_t launch_kcp_compose(const float* trans, int n_prev, const float* init_state, float* state_in, int N, int H,
                               cudaStream_t stream);

// Backward of the chunkwise prefill.  The workspace holds the forward's whole-
// sequence workspace (fwd_bytes: kda_chunk_fwd_workspace_size's bytes_full),
// then chunk_bwd_extra_bytes of chunk-boundary states and state gradients.
size_t chunk_bwd_extra_bytes(int n_seqs, int H, int64_t max_seqlen);
cudaError_t chunk_bwd_launch(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, const void* d_o, const float* d_final, float* dq, float* dk,
                             float* dv, float* dlog_alpha, float* dbeta, float* d_init, int B, int64_t T, int H,
                             const int32_t* cu, int n_seqs, int64_t max_seqlen, bool in_bf16, float scale,
                             void* workspace, size_t fwd_bytes, cudaStream_t stream);

}  // namespace kda
