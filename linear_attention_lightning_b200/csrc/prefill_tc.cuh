// placeholder, replaced by the tcgen05 kernel
#pragma once
#include <string>
#include "common.cuh"
#include "../../include/lightning.h"
namespace la {
inline bool tc_supports(bool bf16, int dim, int block) { (void)bf16; (void)dim; (void)block; return false; }
inline la_status launch_tc(const void*, const void*, const void*, const float*, int, int, int, int,
                           const float*, void*, float*, cudaStream_t, std::string* err) {
    *err = "tcgen05 kernel not built"; return LA_ERR_UNSUPPORTED; }
}
