// The library's single point of entry for device memory, plus host-side fault
// injection for tests (include/ttt_testing.h).
//
// Every device allocation the library makes goes through device_alloc(), so a
// test can make any chosen one of them fail and check that the caller reports
// TTT_ERR_OOM and releases what it already holds; and so the one call site of
// cudaMalloc is easy to audit.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ttt {
// cudaMalloc, unless an injected failure is due (then cudaErrorMemoryAllocation, nothing allocated).
cudaError_t device_alloc(void** p, size_t bytes);
void device_free(void* p);
}  // namespace ttt
