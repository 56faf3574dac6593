// klein.cu -- libklein.so is built as one translation unit so every kernel
// shares the per-device status word without relocatable device code.
#include "kl_quant.cu"
#include "kl_gemm.cu"
#include "kl_attn.cu"
#include "kl_sparse.cu"
#include "kl_vc.cu"
#include "kl_api.cu"
#include "kl_noalloc.cu"
#include "kl_dit.cu"
#include "kl_diag.cu"
