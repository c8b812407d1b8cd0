// kvq_attn_d64.cu -- the decode attention at head dimension D = 64 (kvq_attn.cuh).
#define KVQ_ATTN_D 64
#include "kvq_attn.cuh"
