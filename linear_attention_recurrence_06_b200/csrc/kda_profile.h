// kda_profile.h -- optional per-kernel device timing (a measurement aid).
// While enabled, the launchers bracket each kernel launch with CUDA events on
// the launch stream; kda_profile_read sums the elapsed device time per kernel.
#pragma once
#include <cuda_runtime.h>

namespace kda {
enum ProfKind { PROF_INTRA = 0, PROF_CHAIN = 1, PROF_GATE_NORM = 2, PROF_DECODE = 3, PROF_CHECK = 4, PROF_KCP_COMPOSE = 5,
               PROF_CHAIN_BWD = 6, PROF_INTRA_BWD = 7, PROF_KINDS = 8 };
bool prof_enabled();
void prof_begin(int kind, cudaStream_t stream);
void prof_end(int kind, cudaStream_t stream);
}  // namespace kda
