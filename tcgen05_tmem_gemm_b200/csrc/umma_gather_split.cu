// Tensor-core GEMM for sm_100a: the gather instances of the kernel in
// umma_kernel.cuh for split-K plans (a thin product whose long operand TMA
// cannot describe), compiled in a unit of their own.
#include "umma_kernel.cuh"

namespace dg {

UmmaKernelFn umma_gather_kernel_split(bool fp8) {
    return fp8 ? umma_gemm_kernel<true, true, true> : umma_gemm_kernel<false, true, true>;
}

}  // namespace dg
