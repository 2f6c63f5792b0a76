// internal.h -- host-side helpers shared by the C entry points (api.cu,
// noalloc.cu, selftest.cu): launch counting and validation of a quantized
// weight's descriptor.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>

#include "codec.h"
#include "nf4_tables.h"
#include "qlora.h"

namespace qlora {

// Returns e; when it is cudaSuccess, adds n to the process-wide count of
// kernels the library has launched (qlora_kernel_launches).
cudaError_t counted(cudaError_t e, int n = 1);

// Checks a quantized-weight descriptor before any launch: NULL descriptor,
// shape range (0 <= rows, cols <= 2^31), block sizes, then (for a non-empty
// weight) NULL buffers and 16-byte alignment, in that order.
qlora_status check_tensor(const qlora_nf4_tensor* t);

// The encode kernel's bucket tables (kernel parameter) of one type's tables.
EncodeTables encode_tables(const Nf4Tables& tabs);

// Device address of the library's error flag on the current device (the flag
// qlora_read_device_errors reads); QLORA_ERR_UNSUPPORTED on a non-sm_100 device.
qlora_status device_error_flag(uint32_t** flag);

}  // namespace qlora
