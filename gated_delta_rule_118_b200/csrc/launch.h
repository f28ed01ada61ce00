// launch.h -- internal (C++) interface between the C ABI layer and the kernels.
// Arguments arrive here already validated by gdn2_api.cu.
#pragma once

#include <cuda_runtime.h>

namespace gdn2 {

struct DecodeArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    float *S;
    void *o;
    int B, H, dk, dv;
    bool bf16;
    cudaStream_t stream;
};

struct FwdArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    const float *S0;  // may be null (zero state)
    void *o;
    float *S_T;       // may be null (not written); may alias S0
    int B, T, H, dk, dv;
    bool bf16;
    cudaStream_t stream;
    unsigned int *err;  // device error word
    int num_sms;
};

cudaError_t launch_decode(const DecodeArgs &a);
cudaError_t launch_fwd_simt(const FwdArgs &a);
cudaError_t launch_fwd_tc(const FwdArgs &a);
int fwd_tc_tile(int B, int H, int dv, int num_sms);

}  // namespace gdn2
