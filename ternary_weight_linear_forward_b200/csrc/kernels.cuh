// kernels.cuh -- host-side launchers of libbitlinear's kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace bl {

constexpr int PREP_MAX_GRID = 1024;

// Output modes of the forward kernels.
enum YMode : int { Y_F32 = 0, Y_BF16 = 1, Y_ACC = 2 };

// Combine modes of the block-glue quantiser (match BL_COMBINE_*).
enum Combine : int { C_NONE = 0, C_ADD = 1, C_SILU_MUL = 2 };

struct DevInfo {
    int num_sms;
    int max_smem_optin;
};

// k_prep.cu
size_t quantize_weights_ws_bytes();
cudaError_t launch_quantize_weights(const float* W, long long n, float eps, int8_t* W_t, float* beta, void* ws,
                                    int num_sms, cudaStream_t st);
cudaError_t launch_pack(const int8_t* W_t, long long nwords, uint32_t* W_p, int num_sms, cudaStream_t st);
size_t binarize_weights_ws_bytes();
cudaError_t launch_binarize_weights(const float* W, long long n, int8_t* W_b, float* alpha, float* beta, void* ws,
                                    int num_sms, cudaStream_t st);
cudaError_t launch_pack_bits(const int8_t* W_b, long long nwords, uint32_t* W_p, int num_sms, cudaStream_t st);

// k_act.cu
// rowsum (may be null): the sum of every token's codes, int32 [M]
cudaError_t launch_quant_act(const void* x, bool bf16, long long M, long long K, int8_t* x_q, float* gamma,
                             cudaStream_t st, int* rowsum = nullptr);
cudaError_t launch_quant_act_grouped(const void* x, bool bf16, long long M, long long K, int G, int8_t* x_q,
                                     float* gamma, cudaStream_t st);
cudaError_t launch_quant_act_rms(const float* a, const float* b, int combine, long long M, long long K, float* h,
                                 int8_t* x_q, float* gamma, cudaStream_t st);

// k_gemv.cu  (M <= 64, CUDA cores)
cudaError_t launch_gemv(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                        int N, void* y, YMode mode, const DevInfo& dev, cudaStream_t st);

bool gemv_fused_quant_ok(long long M, long long K);
cudaError_t launch_gemv_fused(const void* x, bool bf16, int M, int K, const uint32_t* W_p, const float* beta, int N,
                              void* y, YMode mode, const DevInfo& dev, cudaStream_t st);
// 1-bit weights (K / 32 words per row), M <= 4 with the x_q staging of the
// fused quantiser; x_dtype 0 fp32, 1 bf16, 2 int8 x_q with gamma
bool gemv_bits_ok(long long M, long long K);
cudaError_t launch_gemv_bits(const void* x, int x_dtype, const float* gamma, int M, int K, const uint32_t* W_p,
                             const float* beta, int N, void* y, YMode mode, const DevInfo& dev, cudaStream_t st);

struct GemvProblem {
    const void* x;
    const float* gamma;  // x is x_q when non-null
    const uint32_t* W_p;
    const float* beta;
    void* y;
    int K, N;
    const int* rowsum;   // with x_q: the row sums of x_q when already known, else null
};
int gemv_group_max();
cudaError_t launch_gemv_fused_group(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode,
                                    const DevInfo& dev, cudaStream_t st);

// k_gemv1.cu  (one token, up to eight problems, CUDA cores, weight stream
// prefetched under the preceding kernel); x_dtype as above
bool gemv1_ok(const GemvProblem* probs, int count, int M, const DevInfo& dev);
cudaError_t launch_gemv1(const GemvProblem* probs, int count, int x_dtype, YMode mode, const DevInfo& dev,
                         cudaStream_t st);

// api.cu: true once after bitlinear_test_expire_next_wait(1) (test hook of
// the bounded waits; consumed by the next launch of the general small-M
// decode kernel)
bool take_wait_expiry_request();

// k_decode_tc.cu  (M <= 16, tcgen05 int8 tensor cores)
int decode_tc_max_m();
bool decode_tc_supported(int M, int K, int N, int count, const DevInfo& dev);
// row tiles per CTA of one swap-AB problem (0 if it does not fit)
int decode_tc_row_tiles(int M, int K, int N, const DevInfo& dev);
cudaError_t launch_decode_tc(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode, const DevInfo& dev,
                             cudaStream_t st);
// api.cu: the kernel that runs a problem set with M tokens under the
// process-wide engine choice
enum DecodePath : int { PATH_CUDA = 0, PATH_TC = 1, PATH_GEMM = 2 };
DecodePath decode_path(int M, const GemvProblem* probs, int count, const DevInfo& dev);
// api.cu: the CUDA-core kernel for a problem set (the one-token streaming
// kernel where it applies and the engine allows it, else the small-M kernels)
cudaError_t launch_decode_cuda(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode,
                               const DevInfo& dev, cudaStream_t st);

// k_gemm.cu  (tcgen05 int8 tensor cores); wbits 2 (trits) or 1 (signs).  The
// workspace holds the row sums and, when few tiles are cut along K
// (allow_split), the per-tile counters and partial tiles; gemm_ws_bytes
// sizes it for allow_split, and M int32 suffice without.
size_t gemm_ws_bytes(long long M, long long N, long long K);
// rowsum_ready: the row sums of x_q are already at the start of ws (written
// by the quantiser), so no row-sum kernel runs.
cudaError_t launch_gemm(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                        int N, void* y, YMode mode, void* ws, const DevInfo& dev, cudaStream_t st, int wbits = 2,
                        bool allow_split = true, bool rowsum_ready = false);

// k_group.cu  (group quantisation along K)
size_t regroup_ws_bytes(long long N, long long K);
cudaError_t launch_regroup(const float* W, long long N, long long K, int G, float* out, int num_sms,
                           cudaStream_t st);
cudaError_t launch_grouped_sum(const float* t, long long t_stride, long long MN, int G, void* y, YMode mode,
                               int num_sms, cudaStream_t st);
cudaError_t launch_grouped_rescale(const int* acc, long long acc_stride, const float* gamma, const float* beta, int M,
                                   int N, int G, void* y, YMode mode, int num_sms, cudaStream_t st);

// Raise a kernel's dynamic shared-memory limit once per device (api.cu).
cudaError_t ensure_smem_optin(const void* kernel, size_t bytes);

// launch helper: every per-token kernel is launched with programmatic stream
// serialisation so it can start while its predecessor drains.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace bl
