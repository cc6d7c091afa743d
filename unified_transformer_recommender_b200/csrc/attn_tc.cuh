#pragma once
#include "common.cuh"
namespace ot {
inline bool tc_attn_supported(const AttnDesc&) { return false; }
inline onetrans_status tc_attn_launch(const AttnDesc&, cudaStream_t) { return ONETRANS_ERR_UNSUPPORTED; }
}
