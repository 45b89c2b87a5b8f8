// launch_util.h -- kernel launch with programmatic dependent launch (PDL).
//
// With FP8Q_PDL (the default), every library kernel is launched with the
// programmatic-stream-serialization attribute and begins with pdl_enter():
// it first waits until the previous grid in the stream has completed and its
// memory is visible (griddepcontrol.wait, so stream order is kept exactly),
// then lets the next grid start launching (griddepcontrol.launch_dependents).
// The next kernel's CTAs can then be placed on SMs while this kernel's last
// CTAs finish, instead of after it.
#pragma once

#include <cuda_runtime.h>

#ifndef FP8Q_PDL
#define FP8Q_PDL 1
#endif

namespace fp8q {

__device__ __forceinline__ void pdl_enter() {
#if FP8Q_PDL
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args... args) {
#if FP8Q_PDL
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
    if (e != cudaSuccess) return e;
#else
    kern<<<grid, block, smem, stream>>>(static_cast<KArgs>(args)...);
#endif
    return cudaGetLastError();
}

}  // namespace fp8q
