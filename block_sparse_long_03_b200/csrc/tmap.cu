// tmap.cu -- host-side creation of TMA tensor maps.  The driver's encoder is
// reached through the runtime's driver entry point, so the library does not
// link against libcuda directly.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc.cuh"

namespace msa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encoder() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
}

}  // namespace

bool make_tmap_bf16(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box) {
    std::call_once(g_encode_once, load_encoder);
    if (g_encode == nullptr || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) {
            st[i] = strides_bytes[i];
            if (st[i] % 16 != 0) return false;
        }
    }
    if (((uintptr_t)base & 15u) != 0) return false;
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                                const_cast<void *>(base), d, st, bx, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace msa
