// sq_lib.cu -- libsq is compiled as one translation unit, so the device status
// word defined in sq_api.cu is shared by every kernel without relocatable
// device code.
#include "sq_api.cu"
#include "sq_quant.cu"
#include "sq_act_variants.cu"
#include "sq_gemm.cu"
#include "sq_probe.cu"
#include "sq_split.cu"
#include "sq_gemm_noalloc.cu"
#include "sq_search.cu"
