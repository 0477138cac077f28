// Single translation unit of libw4a4: every kernel and the C-ABI are
// compiled together so device globals (the error word) are shared without
// relocatable device code.
#include "w4a4_api.cu"
#include "calib.cu"
#include "pack.cu"
#include "prep.cu"
#include "prep_block.cu"
#include "gemm.cu"
#include "noalloc.cu"
#include "checkpoint.cu"
#include "metrics.cu"
#include "ffn.cu"
