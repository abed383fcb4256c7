// host_cache.h -- launch facts cached on the host per CUDA context: the current context's
// identity, the SM count, resident CTAs per SM of a kernel, and the dynamic shared-memory
// limit already raised on a kernel. Every cache is keyed by the context (which identifies the
// device and changes after a device reset) and guarded by a mutex, so one host thread may
// drive several devices and several host threads may launch at once.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qn {

// Identity of the calling thread's current context (0 when none is current or the driver
// cannot tell; callers then key by the device ordinal alone).
uint64_t current_context_id();

// SM count of the current device (cached per context).
cudaError_t device_sm_count(int *sms);

// Resident CTAs per SM of `kern` with `threads` threads and `smem` bytes of dynamic shared
// memory on the current device (cached per context; at least 1).
cudaError_t resident_ctas(const void *kern, int threads, size_t smem, int *ctas);

// Clusters of `cluster` CTAs (`threads` threads, `smem` bytes each) of `kern` that can be
// resident at once on the current device (the query accounts for GPC boundaries; cached per
// context; 0 when none fits).
cudaError_t resident_clusters(const void *kern, int threads, int cluster, size_t smem, int *clusters);

// Raise the dynamic shared-memory limit of `kern` to at least `smem` bytes on the current
// context; the attribute call is made only when a launch needs more than the last one set.
cudaError_t ensure_smem_limit(const void *kern, size_t smem);

}  // namespace qn
