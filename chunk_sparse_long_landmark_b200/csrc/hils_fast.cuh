// hils_fast.cuh -- entry points of the tensor-core / HBM-tuned kernels.
#pragma once

#include "hils_internal.cuh"

namespace hils {

// True when the problem fits the fast kernels' tile set (otherwise the SIMT
// kernels run it).
bool fast_path_supported(const Problem &p);
// True when the selection stage has a tensor-core kernel for the problem.
bool fast_select_supported(const Problem &p);
// Scratch bytes the fast kernels need inside the caller's workspace.
size_t fast_workspace_bytes(const Problem &p);
// Enqueue the fast kernels of one stage (each counts its own launches).
// `ws` is 256-byte aligned, `ws_bytes` as above.
cudaError_t launch_fast_select(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st);
cudaError_t launch_fast_attend(Problem &p, void *ws, size_t ws_bytes,
                               cudaStream_t st);

}  // namespace hils
