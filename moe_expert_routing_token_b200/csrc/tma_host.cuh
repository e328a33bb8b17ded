// Host side of the TMA tensor maps: cuTensorMapEncodeTiled reached through
// the runtime's driver entry point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Encode a 2-D row-major bf16 or fp32 tensor (rows x cols, row stride in
// bytes) with a (box_cols x box_rows) box and 128-byte swizzle.  Returns
// cudaSuccess or the error to report.
cudaError_t encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                           uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                           uint32_t box_cols, uint32_t box_rows, bool swizzle128);

}  // namespace moe
