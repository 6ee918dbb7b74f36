// Decode and prefill kernels for K codes of 3 bits and V codes of 2 bits (explicit instantiation).
#include "iq_prefill_impl.cuh"

namespace iq {
template int launch_decode_kv<3, 2>(const LayerView&, const void*, int, int, int, const int32_t*, int, const float*,
                                   float*, void*, const KernelConsts&, void*, const void*, const void*,
                                   const DeferredInfo*);
template int launch_prefill_kv<3, 2>(const LayerView&, const void*, int, int, int, int, const int32_t*, int,
                                    const float*, float*, void*, const KernelConsts&, void*, int);
}  // namespace iq
