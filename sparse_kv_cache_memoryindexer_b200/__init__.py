"""B200-native hot path of Lookahead Sparse Attention: Memory-Indexer fetch decision plus the
Lightning-Indexer Top-k over the fetched entries.  See include/lsa.h for the C ABI."""
from .lsa import (LSAError, MappedPool, lsa_check_device, lsa_fetch_gather, lsa_fetch_gather_incremental,
                  lsa_fetch_incremental_workspace_size, lsa_lightning_topk, lsa_lightning_topk_step,
                  lsa_lightning_topk_step_workspace_size, lsa_golden_labels,
                  lsa_golden_labels_workspace_size, lsa_indexer_train_step,
                  lsa_indexer_train_workspace_size,
                  lsa_lightning_topk_workspace_size, lsa_memindex_score_select,
                  lsa_memindex_score_select_static, lsa_project,
                  lsa_project_workspace_size, lsa_score_select_workspace_size, lsa_selftest_wait_timeout,
                  launch_count, version)
from .pipeline import IndexerPath

__all__ = ["LSAError", "MappedPool", "IndexerPath", "lsa_check_device", "lsa_fetch_gather",
           "lsa_fetch_gather_incremental", "lsa_fetch_incremental_workspace_size",
           "lsa_lightning_topk", "lsa_lightning_topk_workspace_size", "lsa_lightning_topk_step",
           "lsa_lightning_topk_step_workspace_size", "lsa_golden_labels", "lsa_golden_labels_workspace_size",
           "lsa_indexer_train_step", "lsa_indexer_train_workspace_size", "lsa_memindex_score_select",
           "lsa_memindex_score_select_static",
           "lsa_project", "lsa_project_workspace_size", "lsa_score_select_workspace_size",
           "lsa_selftest_wait_timeout", "launch_count", "version"]
