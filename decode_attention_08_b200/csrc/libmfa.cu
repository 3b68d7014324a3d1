// libmfa.cu -- single translation unit of libmfa.so (one module, so the
// per-device status word needs no relocatable device code).
#include "decode_kernel.cu"
#include "qproj_kernel.cu"
#include "merge_kernel.cu"
#include "mfa_api.cu"
