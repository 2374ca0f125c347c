// Test helper: evaluates the sampler's own fp64 exp (exp_neg) and CUDA's exp
// on the same arguments so the test can bound its error in ulps.
#include "../../verify_step_lm_b200/csrc/sampler.cu"

__global__ void exp_pair_kernel(const double *x, double *mine, double *ref, int n) {
    __shared__ double tab[mtpv::kExpTab];
    mtpv::build_exp_table(tab);
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        mine[i] = mtpv::exp_neg(x[i], tab);
        ref[i] = exp(x[i]);
    }
}

extern "C" int exp_pair(const double *x, double *mine, double *ref, int n) {
    exp_pair_kernel<<<(n + 255) / 256, 256>>>(x, mine, ref, n);
    return (int)cudaDeviceSynchronize();
}
