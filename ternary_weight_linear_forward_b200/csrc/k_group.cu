// k_group.cu -- group quantisation: the weight regrouping copy and the
// per-group rescale.
//
// unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
// auf lokale Geraete", section "Gruppenquantisierung und -normalisierung":
// weights and activations are divided into G groups whose parameters are
// computed independently.  The groups are G contiguous, equal blocks of the
// contraction dimension K, so group g owns W[:, K_g] with its absmean beta_g
// and x[m, K_g] with its absmax gamma_{m,g}; the integer contraction of each
// group is rescaled by its own beta_g * gamma_{m,g} / Q_b (eq. 3) and the
// binary32 terms are added in increasing g.
//
// Storage is group-major ([G][N][K/G] weights, [G][M][K/G] codes), so every
// group is an ordinary matrix for the existing quantisation, packing and
// contraction kernels; only the passes below are particular to groups.
#include "common.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int GROUP_THREADS = 256;

// out[g][n][j] = W[n][g * Kg + j], in float4 units (Kg % 4 == 0).
__global__ void __launch_bounds__(GROUP_THREADS) regroup_kernel(const float4* __restrict__ W, long long N, int K,
                                                                int G, float4* __restrict__ out) {
    const int Kg4 = K / G / 4, K4 = K / 4;
    const long long per_group = N * Kg4, total = per_group * G;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long g = i / per_group, r = i % per_group;
        const long long n = r / Kg4, j = r % Kg4;
        out[i] = __ldg(&W[n * K4 + g * Kg4 + j]);
    }
}

// y[m, n] = sum over g = 0, 1, ... of (float)acc[g][m][n] * ((beta_g * gamma[m][g]) / 127),
// each term and each add one binary32 operation, in increasing g.  Group g's
// accumulators start at acc + g * acc_stride.
__global__ void __launch_bounds__(GROUP_THREADS) grouped_rescale_kernel(const int* __restrict__ acc,
                                                                        long long acc_stride,
                                                                        const float* __restrict__ gamma,
                                                                        const float* __restrict__ beta, int M, int N,
                                                                        int G, void* __restrict__ y, int mode) {
    pdl_launch_dependents();
    pdl_wait();
    const long long MN = (long long)M * N;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < MN;
         i += (long long)gridDim.x * blockDim.x) {
        const long long m = i / N;
        float v = 0.0f;
        for (int g = 0; g < G; ++g) {
            const float f = __fdiv_rn(__fmul_rn(__ldg(beta + g), __ldg(gamma + m * G + g)), 127.0f);
            const float t = __fmul_rn((float)__ldcg(acc + g * acc_stride + i), f);
            v = g == 0 ? t : __fadd_rn(v, t);
        }
        if (mode == Y_F32)
            reinterpret_cast<float*>(y)[i] = v;
        else
            reinterpret_cast<uint16_t*>(y)[i] = f32_to_bf16_rn(v);
    }
}

// y[m, n] = t_0 + t_1 + ... + t_{G-1} in binary32, in increasing g, where
// group g's terms t_g (already rescaled) start at t + g * t_stride.
__global__ void __launch_bounds__(GROUP_THREADS) grouped_sum_kernel(const float* __restrict__ t, long long t_stride,
                                                                    long long MN, int G, void* __restrict__ y,
                                                                    int mode) {
    pdl_launch_dependents();
    pdl_wait();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < MN;
         i += (long long)gridDim.x * blockDim.x) {
        float v = __ldcg(t + i);
        for (int g = 1; g < G; ++g) v = __fadd_rn(v, __ldcg(t + g * t_stride + i));
        if (mode == Y_F32)
            reinterpret_cast<float*>(y)[i] = v;
        else
            reinterpret_cast<uint16_t*>(y)[i] = f32_to_bf16_rn(v);
    }
}

}  // namespace

cudaError_t launch_grouped_sum(const float* t, long long t_stride, long long MN, int G, void* y, YMode mode,
                               int num_sms, cudaStream_t st) {
    const int grid =
        (int)std::max<long long>(1, std::min<long long>((MN + GROUP_THREADS - 1) / GROUP_THREADS, (long long)num_sms * 8));
    return launch_pdl(grouped_sum_kernel, dim3(grid), dim3(GROUP_THREADS), 0, st, t, t_stride, MN, G, y, (int)mode);
}

size_t regroup_ws_bytes(long long N, long long K) { return (size_t)(N * K * 4 + 255) / 256 * 256; }

cudaError_t launch_regroup(const float* W, long long N, long long K, int G, float* out, int num_sms,
                           cudaStream_t st) {
    const long long n4 = N * K / 4;
    const int grid = (int)std::max<long long>(1, std::min<long long>((n4 + GROUP_THREADS - 1) / GROUP_THREADS,
                                                                     (long long)num_sms * 8));
    regroup_kernel<<<grid, GROUP_THREADS, 0, st>>>(reinterpret_cast<const float4*>(W), N, (int)K, G,
                                                   reinterpret_cast<float4*>(out));
    return cudaGetLastError();
}

cudaError_t launch_grouped_rescale(const int* acc, long long acc_stride, const float* gamma, const float* beta, int M,
                                   int N, int G, void* y, YMode mode, int num_sms, cudaStream_t st) {
    const long long MN = (long long)M * N;
    const int grid =
        (int)std::max<long long>(1, std::min<long long>((MN + GROUP_THREADS - 1) / GROUP_THREADS, (long long)num_sms * 8));
    return launch_pdl(grouped_rescale_kernel, dim3(grid), dim3(GROUP_THREADS), 0, st, acc, acc_stride, gamma, beta, M,
                      N, G, y, (int)mode);
}

}  // namespace bl
