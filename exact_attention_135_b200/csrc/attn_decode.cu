// Paged MLA decode (MQA-absorb form): split-KV kernel plus LSE combine.
#include "host_common.h"

extern "C" size_t attn_decode_paged_workspace_size(int B, int Hq, int Dv) {
  (void)B;
  (void)Hq;
  (void)Dv;
  return 0;
}

extern "C" int attn_decode_paged(const void* q, const void* kv_pages, const int32_t* block_table,
                                 const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Dk, int Dv,
                                 int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return ATTN_ERR_UNSUPPORTED;
}
