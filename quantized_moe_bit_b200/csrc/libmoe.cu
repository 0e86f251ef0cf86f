// Single translation unit of the CUDA part of libmoe (the kernels share
// device symbols such as the check word without relocatable device code).
#include "kernels.cu"
#include "api.cu"
#include "expert_noalloc.cu"
#include "ep.cu"
