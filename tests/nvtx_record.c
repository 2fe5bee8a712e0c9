/* NVTX injection library for tests/test_gpu_nvtx.py: records every range push
 * and pop of the process in the file named by QFP4_NVTX_LOG. NVTX loads it
 * from NVTX_INJECTION64_PATH and calls InitializeInjectionNvtx2, which points
 * the core module's RangePushA / RangePop slots at the recorders below. */
#include <stdio.h>
#include <stdlib.h>

#include <nvtx3/nvToolsExt.h>

static FILE* g_log;

static int record_push(const char* message) {
    if (g_log) {
        fprintf(g_log, "push %s\n", message ? message : "");
        fflush(g_log);
    }
    return 0;
}

static int record_pop(void) {
    if (g_log) {
        fputs("pop\n", g_log);
        fflush(g_log);
    }
    return 0;
}

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_export_table) {
    const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_export_table(NVTX_ETID_CALLBACKS);
    NvtxFunctionTable table = 0;
    unsigned int size = 0;
    if (cb == NULL || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size)) return 0;
    if (size <= NVTX_CBID_CORE_RangePop) return 0;
    const char* path = getenv("QFP4_NVTX_LOG");
    g_log = path ? fopen(path, "w") : NULL;
    *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)record_push;
    *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)record_pop;
    return 1;
}
