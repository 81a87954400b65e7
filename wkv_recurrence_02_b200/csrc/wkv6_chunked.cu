// wkv6_chunked.cu -- chunked WKV-6 prefill (tensor-core kernel lands here).
#include "wkv_internal.cuh"

namespace wkv {

cudaError_t wkv6_chunked_launch(const Wkv6Args &a, cudaStream_t s)
{
    return wkv6_serial_launch(a, s);
}

}  // namespace wkv
