// Host-side declarations shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sharq.h"

namespace sq {

struct LaunchCtx {
    cudaStream_t stream;
    unsigned *status;      // device status word
    uint64_t wait_ns;      // bound of every device-side wait
    int num_sms;
    int launches;          // kernels enqueued by the current entry point
};

// norm: 0 = LayerNorm, 1 = RMSNorm (beta must be NULL).
sharq_status launch_prepare(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma,
                            const void *beta, float eps, int norm);
// The pair-wise 4:8 mode (P from prep_layout_sparse).
sharq_status launch_prepare_sparse(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma,
                                   const void *beta, float eps, int norm);
// x_out = RN16(h + d), then the preparation of x_out (P from prep_layout).
sharq_status launch_prepare_add(LaunchCtx &ctx, const sharq_prep &P, const void *h, const void *d, void *x_out,
                                const void *gamma, const void *beta, float eps, int norm);
sharq_status launch_prepare_grouped(LaunchCtx &ctx, const sharq_prep &P, const void *x, int64_t rows,
                                    const int32_t *offsets, int32_t groups, const void *gamma, const void *beta,
                                    float eps, int norm);
sharq_status launch_quantize_weight(LaunchCtx &ctx, const sharq_wq &W, const void *w, int64_t groups,
                                   int64_t gstride);
sharq_status launch_quantize_weight_fused(LaunchCtx &ctx, const sharq_wq &W, const void *w, const int64_t *seg_rows,
                                         int n_segs);
// bias: fp16 [n_out] or NULL
sharq_status launch_linear(LaunchCtx &ctx, const sharq_prep &P, const sharq_wq &W, const void *bias, void *out);
sharq_status launch_linear_grouped(LaunchCtx &ctx, const sharq_prep &P, const sharq_wq &W, const int32_t *offsets,
                                   int32_t groups, int64_t rows, int64_t w_gstride, void *out);
sharq_status launch_gather(LaunchCtx &ctx, const sharq_prep &S, const int32_t *row_idx, const int32_t *offsets,
                           int32_t groups, int64_t rows, const sharq_prep &D);
sharq_status launch_wait_probe(LaunchCtx &ctx, uint64_t limit_ns);
// Records the kernel count that sharq_last_launch_count reports.
void note_launches(int n);
sharq_status launch_div_check(LaunchCtx &ctx, uint64_t count, uint64_t seed, uint64_t *mismatches, float *examples);

}  // namespace sq

#define SQ_CUDA_TRY(expr)                                         \
    do {                                                          \
        cudaError_t _e = (expr);                                  \
        if (_e != cudaSuccess) return SHARQ_ERR_CUDA;             \
    } while (0)
