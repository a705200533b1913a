// hybattn.cu -- single translation unit of libhybattn.so (keeps the device
// status word and every kernel in one module without relocatable device code).
#include "compress.cu"
#include "fp4.cu"
#include "index_topk.cu"
#include "index_tc.cu"
#include "attn.cu"
#include "attn_dense.cu"
#include "attn_sparse.cu"
#include "decode_append.cu"
#include "gated.cu"
#include "backward.cu"
#include "api.cu"
#include "noalloc.cu"
