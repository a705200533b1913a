// hybattn.cu -- single translation unit of libhybattn.so (keeps the device
// status word and every kernel in one module without relocatable device code).
#include "compress.cu"
#include "index_topk.cu"
#include "attn.cu"
#include "api.cu"
#include "noalloc.cu"
