// page_allocator.cu -- host-side page allocator of the C ABI (no GPU work).
//
// Physical pages of the shared pool belong to one sequence at a time and go
// back to the pool when it ends (comrad404 article on samir-vllm, section
// "Что README говорит о KV-кэше и пакетном декодировании", which lists block
// tables and page freeing beside batched decode).  Continuous batching admits
// a queued request only if the page budget fits, lets requests that do not
// fit wait in arrival order, and rejects a request whose budget exceeds the
// whole pool ("Curso gratuito recorre la inferencia de LLM...", section on
// how the engine manages the KV-cache memory).  This file is the page-level
// part of that: all-or-nothing allocation from a LIFO free stack, with
// distinct errors for "not enough free pages now" (queue) and "more pages
// than the pool has" (reject).
#include <new>
#include <vector>

#include "pkv.h"

struct pkv_page_allocator {
  std::vector<int32_t> free_stack;   // top = back
  std::vector<uint8_t> in_use;       // per page
};

extern "C" {

int pkv_allocator_create(int32_t num_pages, pkv_page_allocator** out) {
  if (!out || num_pages < 1) return PKV_ERR_INVALID_ARG;
  *out = nullptr;
  pkv_page_allocator* a = new (std::nothrow) pkv_page_allocator();
  if (!a) return PKV_ERR_INVALID_ARG;
  try {
    a->free_stack.resize(num_pages);
    a->in_use.assign(num_pages, 0);
  } catch (...) {
    delete a;
    return PKV_ERR_INVALID_ARG;
  }
  for (int32_t i = 0; i < num_pages; ++i) a->free_stack[i] = num_pages - 1 - i;  // page 0 on top
  *out = a;
  return PKV_OK;
}

int pkv_allocator_destroy(pkv_page_allocator* a) {
  delete a;
  return PKV_OK;
}

int32_t pkv_allocator_free_count(const pkv_page_allocator* a) {
  return a ? static_cast<int32_t>(a->free_stack.size()) : -1;
}

int pkv_allocator_alloc(pkv_page_allocator* a, int32_t count, int32_t* pages_out) {
  if (!a || count < 0 || (count > 0 && !pages_out)) return PKV_ERR_INVALID_ARG;
  if (static_cast<size_t>(count) > a->in_use.size()) return PKV_ERR_TOO_LARGE;
  if (static_cast<size_t>(count) > a->free_stack.size()) return PKV_ERR_OUT_OF_PAGES;
  for (int32_t i = 0; i < count; ++i) {
    const int32_t p = a->free_stack.back();
    a->free_stack.pop_back();
    a->in_use[p] = 1;
    pages_out[i] = p;
  }
  return PKV_OK;
}

int pkv_allocator_free(pkv_page_allocator* a, const int32_t* pages, int32_t count) {
  if (!a || count < 0 || (count > 0 && !pages)) return PKV_ERR_INVALID_ARG;
  const int32_t n = static_cast<int32_t>(a->in_use.size());
  // validate everything first: nothing is freed if any page is bad
  std::vector<uint8_t> seen;
  for (int32_t i = 0; i < count; ++i) {
    const int32_t p = pages[i];
    if (p < 0 || p >= n || !a->in_use[p]) return PKV_ERR_INVALID_ARG;
    if (seen.empty()) seen.assign(n, 0);
    if (seen[p]) return PKV_ERR_INVALID_ARG;   // listed twice
    seen[p] = 1;
  }
  for (int32_t i = 0; i < count; ++i) {
    a->in_use[pages[i]] = 0;
    a->free_stack.push_back(pages[i]);
  }
  return PKV_OK;
}

}  // extern "C"
