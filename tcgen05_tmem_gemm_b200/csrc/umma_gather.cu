// Tensor-core GEMM for sm_100a: the gather instances of the kernel in
// umma_kernel.cuh (cp.async producer warps for an operand TMA cannot
// describe), compiled apart from the direct-load ones.
#include "umma_kernel.cuh"

namespace dg {

UmmaKernelFn umma_gather_kernel(bool fp8) {
    return fp8 ? umma_gemm_kernel<true, true> : umma_gemm_kernel<false, true>;
}

}  // namespace dg
