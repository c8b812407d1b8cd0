// kvq_attn_d128.cu -- the decode attention at head dimension D = 128 (kvq_attn.cuh).
#define KVQ_ATTN_D 128
#include "kvq_attn.cuh"
