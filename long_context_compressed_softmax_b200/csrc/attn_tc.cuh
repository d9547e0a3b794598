#pragma once
#include "common.cuh"
namespace lcsa {
static bool attn_tc_supported(const lcsa_attn_args*) { return false; }
static size_t attn_tc_workspace(const lcsa_attn_args*, int) { return 0; }
static cudaError_t launch_attn_tc(const lcsa_attn_args*, int, void*, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace lcsa
