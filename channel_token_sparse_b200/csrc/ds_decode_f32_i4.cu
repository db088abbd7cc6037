// Instantiations of the fused decode kernel for k/v dtype f32, label kind i4.
#include "ds_decode_kernel.cuh"
#include "ds_internal.h"

namespace ds {

DecodeKernel decode_kernel_f32_i4(int D, int C, int GT) {
#define DS_K(D_, C_, G_) \
    if (D == D_ && C == C_ && GT == G_) return &ds_decode_kernel<float, 1, D_, C_, G_, false>;
#define DS_KG(D_, C_) DS_K(D_, C_, 1) DS_K(D_, C_, 2) DS_K(D_, C_, 4) DS_K(D_, C_, 8)
    DS_KG(64, 8) DS_KG(64, 16) DS_KG(64, 32) DS_KG(64, 64)
    DS_KG(128, 8) DS_KG(128, 16) DS_KG(128, 32) DS_KG(128, 64) DS_KG(128, 128)
#undef DS_KG
#undef DS_K
    return nullptr;
}

}  // namespace ds
