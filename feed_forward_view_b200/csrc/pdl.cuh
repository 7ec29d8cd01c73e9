// pdl.cuh -- programmatic dependent launch for the library's kernels.
//
// A kernel launched with launch_pdl may be scheduled while the work before it
// in the stream is still finishing, so that its CTAs are dispatched during the
// previous kernel's last wave instead of after it. Such a kernel must run
// griddep_wait() before it reads or writes global memory that earlier work may
// touch. Every kernel of the library starts with griddep_wait(), so that only
// the launch itself overlaps: everything the kernel does happens after the
// preceding work has finished and its writes are visible, exactly as with an
// ordinary launch. griddep_launch_dependents() lets the next kernel be
// scheduled once every CTA of this one has issued it: the attention kernels
// issue it first thing (their grids are often a single wave, whose free SMs
// the next kernel can then take at once), the memory-bound kernels at the end
// of each CTA's work (their grids are many waves, and an early signal only
// parks the next kernel's CTAs, waiting, through most of this one: measured
// slower at 274 800 tokens). Both instructions do nothing when there is no
// programmatic dependency (an ordinary launch, or nothing before it).
#pragma once

#include <utility>

#include <cuda_runtime.h>

namespace vggt {

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// kernel<<<grid, block, smem, stream>>>(args...), allowed to start while the
// stream's previous kernel finishes (see above). Returns the launch's error.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace vggt
