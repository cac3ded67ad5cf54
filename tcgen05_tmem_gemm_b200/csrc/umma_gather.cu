// Tensor-core GEMM for sm_100a: the gather instances of the kernel in
// umma_kernel.cuh (cp.async producer warps for an operand TMA cannot
// describe) for unsplit plans, compiled apart from the direct-load ones.
#include "umma_kernel.cuh"

namespace dg {

UmmaKernelFn umma_gather_kernel_unsplit(bool fp8) {
    return fp8 ? umma_gemm_kernel<true, true, false> : umma_gemm_kernel<false, true, false>;
}

UmmaKernelFn umma_gather_kernel(bool fp8, bool split) {
    return split ? umma_gather_kernel_split(fp8) : umma_gather_kernel_unsplit(fp8);
}

}  // namespace dg
