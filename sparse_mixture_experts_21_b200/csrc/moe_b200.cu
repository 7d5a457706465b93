// Single translation unit of the library (one module, so every kernel file sees
// the same device status word without relocatable device code).
#include "tmap.cu"
#include "capi.cu"
#include "route.cu"
#include "permute.cu"
#include "permute_noalloc.cu"
#include "ffn_tc.cu"
#include "ffn_f32.cu"
#include "combine_stats.cu"
#include "expert_choice.cu"
#include "ffn_fp8.cu"
#include "ffn_mx.cu"
#include "ep.cu"
