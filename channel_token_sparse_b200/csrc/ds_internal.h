// ds_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ds {

struct DecodeParams;
using DecodeKernel = void (*)(const DecodeParams);

// Kernel instantiation for (k/v dtype, label kind, D, C, GT); nullptr if absent.
DecodeKernel decode_kernel_f32_fp(int D, int C, int GT);
DecodeKernel decode_kernel_f32_i4(int D, int C, int GT);
DecodeKernel decode_kernel_bf16_fp(int D, int C, int GT);
DecodeKernel decode_kernel_bf16_i4(int D, int C, int GT);
// The same for paged K/V pools (ds_decode_step_paged).
DecodeKernel decode_kernel_f32_fp_paged(int D, int C, int GT);
DecodeKernel decode_kernel_f32_i4_paged(int D, int C, int GT);
DecodeKernel decode_kernel_bf16_fp_paged(int D, int C, int GT);
DecodeKernel decode_kernel_bf16_i4_paged(int D, int C, int GT);

// Process-unique id of the current CUDA context (false if there is none):
// the key of the per-context caches of __device__ variable addresses.
bool current_context_id(unsigned long long* id);

struct LabelArgs {
    const void* k;
    bool kdt_bf16;
    bool int4;
    const int32_t* idx;
    int b, hkv, t_begin, t_end, s_cap, d, c;
    void* label;
    uint16_t* lscale;
    uint16_t* lzero;
    const int32_t* block_table = nullptr;  // paged key cache (see ds_label.cu)
    int max_blocks = 0, page_shift = 0, num_blocks = 0;
    unsigned int* err = nullptr;  // device word recording a bounded wait that gave up (pipelined build)
    int sms = 148;                // SMs of the device (pipelined build grid)
};
cudaError_t launch_label(const LabelArgs& a, cudaStream_t st);

// Channel ranking criteria (values of ds_calib_criterion).
enum { kCritLeanK = 0, kCritQ = 1, kCritK = 2, kCritQK = 3, kCritQKChunked = 4 };

struct CalibArgs {
    const void* q_win;
    const void* k;
    bool bf16;
    int n, hq, hkv, w, s, d, c;
    float* ratio;
    int32_t* idx;
    void* ws;
    int criterion = kCritLeanK;
    int chunk = 0;  // context chunk length (kCritQKChunked only)
};
size_t calib_workspace_bytes(int n, int hkv, int d);
cudaError_t launch_calib(const CalibArgs& a, cudaStream_t st);
// Same launch with the scratch taken from a fixed device array (no allocation).
size_t calib_static_scratch_bytes();
cudaError_t launch_calib_static(CalibArgs a, cudaStream_t st);

}  // namespace ds
