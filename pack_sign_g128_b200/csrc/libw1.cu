// Single translation unit for libw1 (the device status word is shared by all
// kernels without relocatable device code).
#include "w1_api.cu"
#include "pack.cu"
#include "gemv.cu"
#include "gemv_tc.cu"
#include "gemv_direct.cu"
#include "sign_gemm.cu"
#include "gemm.cu"
#include "dbf_tc.cu"
#include "dbf.cu"
#include "moe.cu"
#include "okt.cu"
#include "measure.cu"
