"""ParaGRU / ParaLSTM parallel-in-time Newton solve for B200 (sm_100a)."""
