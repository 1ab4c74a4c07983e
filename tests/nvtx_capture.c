/* nvtx_capture.c -- a minimal NVTX tool for the tests: loaded through
 * NVTX_INJECTION64_PATH, it takes over the core range push / pop calls of
 * every NVTX instance in the process and appends one line per call to the
 * file named by HYQ_NVTX_LOG ("push <name>" or "pop").  Test infrastructure
 * only; built by tests/test_nvtx.py with the host compiler. */
#include <nvtx3/nvToolsExt.h>
#include <stdio.h>
#include <stdlib.h>

static FILE *log_file;

static int capture_push(const char *name) {
  if (log_file) {
    fprintf(log_file, "push %s\n", name ? name : "");
    fflush(log_file);
  }
  return 0;
}

static int capture_pop(void) {
  if (log_file) {
    fputs("pop\n", log_file);
    fflush(log_file);
  }
  return 0;
}

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks *cb = (const NvtxExportTableCallbacks *)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = 0;
  unsigned int last = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &last) || last < NVTX_CBID_CORE_RangePop)
    return 0;
  if (!log_file) {
    const char *path = getenv("HYQ_NVTX_LOG");
    log_file = path ? fopen(path, "a") : NULL;
  }
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)capture_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)capture_pop;
  return 1;
}
