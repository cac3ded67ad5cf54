// Tensor-core GEMM for sm_100a: the direct-load instances of the kernel in
// umma_kernel.cuh (TMA for both operands) and the launcher.  The gather
// instances are compiled apart, in umma_gather.cu (unsplit plans) and
// umma_gather_split.cu (split-K plans).
#include "umma_kernel.cuh"

namespace dg {

size_t umma_smem_bytes(int bn, int stages, bool gather, bool epi_tma, int split) {
    return smem_layout(bn, stages, gather, epi_tma, split).total;
}

uint32_t umma_split_out_bytes(int bn, int split) { return split_out_bytes(bn, split); }

int umma_max_stages(int bn, bool gather, bool epi_tma, int split) {
    int s = 2;
    while (s < 12 && smem_layout(bn, s + 1, gather, epi_tma, split).total <= 227 * 1024) ++s;
    return s;
}

cudaError_t launch_umma(const UmmaParams &p, const CUtensorMap *tp, const CUtensorMap *tq, const CUtensorMap *tc,
                        bool fp8, bool gather, int grid, size_t smem, cudaStream_t s) {
    const bool split = p.split_k > 1;
    UmmaKernelFn kern;
    if (gather) kern = umma_gather_kernel(fp8, split);
    else kern = fp8 ? umma_gemm_kernel<true, false, true> : umma_gemm_kernel<false, false, true>;
    // raise the kernel's dynamic shared-memory limit once per device and size, not per call
    static SmemLimit s_limit[6];
    const cudaError_t e = s_limit[(fp8 ? 3 : 0) + (gather ? (split ? 2 : 1) : 0)].ensure(kern, smem);
    if (e != cudaSuccess) return e;
    const int cluster = (p.split_k > 1 && !p.red_add) ? p.split_k
                                                        : (gather && p.gather_cluster > 1 ? p.gather_cluster : 1);
    return launch_ex(kern, dim3(grid), dim3(gather ? 448 : 192), smem, s, dim3(cluster, 1, 1), p.pdl, *tp, *tq, *tc,
                     p);
}

}  // namespace dg
