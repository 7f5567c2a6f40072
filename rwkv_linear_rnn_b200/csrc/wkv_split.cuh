// wkv_split.cuh -- shared definitions of the summary / prefix / replay
// forward (internal).
#pragma once

#include "wkv_internal.cuh"

namespace wkv {

constexpr int kS3Chunk = 64;  // tokens per chunk (== checkpoint interval)
constexpr int kS3Batch = 16;  // rows per load batch
static_assert(kS3Chunk == kCkpt, "chunk starts are the checkpoints");

struct Scan3Args {
  FwdArgs f;
  float *sums;   // [npos][4][nchains][32]: chunk summaries (anchored exponent)
  float *carry;  // [npos][3][B][C]: state at each chunk start (checkpoint format)
  int64_t npos;  // chunks per chain
};

cudaError_t launch_fwd_prefix(const Scan3Args &a, cudaStream_t st);

}  // namespace wkv
