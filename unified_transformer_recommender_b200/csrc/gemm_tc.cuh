#pragma once
#include "common.cuh"
namespace ot {
inline bool tc_gemm_supported(const GemmDesc&) { return false; }
inline onetrans_status tc_gemm_launch(const GemmDesc&, cudaStream_t) { return ONETRANS_ERR_UNSUPPORTED; }
}
