#include "wq_internal.h"
namespace wq {
wq_status launch_gemm(const Problem&, cudaStream_t) { return WQ_ERR_UNSUPPORTED; }
wq_status gemm_device_status(int) { return WQ_OK; }
}
