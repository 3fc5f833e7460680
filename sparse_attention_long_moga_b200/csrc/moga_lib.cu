// Single translation unit of the MoGA sm_100a library (one device error word,
// no relocatable device code needed).
#include "api_common.cu"
#include "route.cu"
#include "permute.cu"
#include "permute_noalloc.cu"
#include "mean_loss.cu"
#include "attention.cu"
#include "attention_bwd.cu"
#include "route_bwd.cu"
#include "sp.cu"
#include "qkv_route.cu"
