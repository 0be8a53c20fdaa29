// Single translation unit of the library: the device status word and wait limit
// are shared by every kernel without relocatable device code.
#include "layer.cu"
#include "select.cu"
#include "score.cu"
#include "gemm_tc.cu"
#include "attention.cu"
#include "abi.cu"
#include "static_ws.cu"
#include "kl_lock.cu"
#include "slowfast.cu"
